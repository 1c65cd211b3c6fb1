// MoBA own-block attention + merge, and the mask-based form, on the 5th-generation tensor
// cores (tcgen05 + TMEM + TMA), one 128-token query tile of one head per CTA and two CTAs per
// SM.  (The past blocks are in attn_past.cu.)
//
// Two modes share the kernel:
//   own  : a row's past partials are merged FIRST: they become the starting state (m, l, O)
//          of the online softmax, which then runs over the block's keys up to the diagonal
//          (causal mask on the diagonal chunk) and ends with the final O (bf16) and LSE.
//   naive: the mask-based form of the same attention (MoBA README, "Implementation
//          Details": moba_naive builds the block mask and runs masked attention): every
//          causal key of the sequence is scored and a row's keys outside its selected blocks
//          get zero weight.  Dense causal cost: a baseline only.
// (youleyou.com,
// "Kimi发布MoBA突破性实现无限上下文", section "PyTorch实现关键要点": attention runs on the
// own block and on the selected blocks separately and the results are merged by online
// softmax; zhuoshang.net, "MoBA是什么？…", section "MoBA的技术原理": causal mask inside the
// current block.)
//
// Per 128-key chunk j:
//   S = Q K_j^T   (tcgen05 SS MMA, fp32 in TMEM)
//   softmax of S in registers (one thread per row = TMEM lane), P (bf16) written back over
//   the first half of S's TMEM columns
//   O += P V_j    (tcgen05 TS MMA, A read from TMEM, fp32 accumulator in TMEM)
// A tile's steps are serial (S, softmax, PV, next S), so one CTA keeps the tensor core busy
// about half the time; the second CTA on the SM fills the other half, and each CTA's set-up,
// merge prologue and epilogue run while the other one computes.  That is why a CTA takes one
// tile (256 TMEM columns, 96 KB of shared memory at D = 128, 192 threads of at most 168
// registers) rather than two tiles in lockstep: two lockstep tiles need the whole SM, and
// their fixed per-CTA costs then leave the tensor core idle.
// Warp roles: warps 0-3 softmax + epilogue, warp 4 TMA producer (Q, then K/V chunks), warp 5
// TMEM owner + MMA issuer (the whole warp runs the issue loop; one elected lane issues).
#include <cudaTypedefs.h>
#include <float.h>

#include "attn_common.cuh"

namespace moba {

namespace {

constexpr int kOwnThreads = 192;
constexpr uint32_t kOwnTmemCols = 256;
constexpr uint32_t kOwnColS = 0;    // S (P aliased on its first 64 columns)
constexpr uint32_t kOwnColO = 128;  // O accumulator

template <int D>
struct OwnLayout {
  static constexpr int kTile = kRows * D * 2;   // bytes of a [128 x D] bf16 tile
  static constexpr int kStages = D == 64 ? 2 : 1;  // K/V stages (two CTAs per SM)
  static constexpr int kQ = 0;
  static constexpr int kK0 = kQ + kTile;
  static constexpr int kV0 = kK0 + kStages * kTile;
  static constexpr int kBar = kV0 + kStages * kTile;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
};
static_assert(2 * (OwnLayout<128>::kAlloc + 1024) <= 228 * 1024, "two CTAs per SM at D = 128");

enum OwnBar { oQFull = 0, oKFull0, oKFull1, oKEmpty0, oKEmpty1, oVFull0, oVFull1, oVEmpty0, oVEmpty1,
              oSFull, oPFull, oOFull, oDone, oNumBars };

template <int D, bool kNaive>
__global__ void __launch_bounds__(kOwnThreads, 2)
    attn_own_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  using L = OwnLayout<D>;
  constexpr int kSt = L::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + oNumBars * 8);
  const Geom& g = a.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ------------------------------------------------------------- work item
  // Own mode: items run sequence by sequence and block by block; inside a block the longest
  // tiles (the last ones, up to 16 chunks) start first, and the heads of a tile run side by
  // side, so a block's K/V chunks serve its tiles and the G heads of each KV group through
  // L2.  Naive mode: the work grows with the block index, so the grid runs backwards.
  const int per_blk = g.bs / kRows;
  int64_t id = kNaive ? (int64_t)gridDim.x - 1 - blockIdx.x : (int64_t)blockIdx.x;
  const int h = (int)(id % g.Hq);
  id /= g.Hq;
  const int qt = per_blk - 1 - (int)(id % per_blk);
  id /= per_blk;
  const int i_blk = (int)(id % g.MB);
  const int s = (int)(id / g.MB);
  const int32_t ts = seq_start(g, s), te = seq_end(g, s);
  const int32_t q0 = ts + i_blk * g.bs + qt * kRows;
  if (q0 >= te) return;
  const int nrows = min(kRows, te - q0);
  // naive mode: every earlier block's chunks come first
  const int before = kNaive ? i_blk * (g.bs / kBN) : 0;
  const int diag = before + qt;  // the diagonal chunk (the last one)
  const int nchunks = diag + 1;
  const int gk = h / g.G;
  const int32_t key0 = kNaive ? ts : ts + i_blk * g.bs;

  // ------------------------------------------------------------- early loads
  // Each softmax thread reads its row's selection and the LSEs of its past partials before
  // the setup below.  The chosen past blocks fill slots 1..np of the row (the selection's
  // padding is at the end), so partial q of the row has the id (row * (top_k - 1) + q).
  int np = 0;
  float pmax = -INFINITY;  // largest past LSE, log2 units
  bool folded = false;     // the row's partials come folded (one partial in mo/mlse)
  if (!kNaive && warp < 4 && tid < nrows) {
    const int64_t qrow = (int64_t)(q0 + tid) * g.Hq + h;
    // The row's partial O rows are read after the setup below; their fetch into L2 starts
    // now, before the selection is known (every slot's row exists; unused ones cost only L2).
    {
      const char* p0 = reinterpret_cast<const char*>(a.part_o + qrow * (g.k - 1) * D);
      const int nq = a.premerged ? 1 : g.k - 1;
      for (int q = 0; q < nq; ++q)
#pragma unroll
        for (int off = 0; off < D * 2; off += 128) prefetch_l2(p0 + q * D * 2 + off);
      if (a.premerged) {
        const char* m0 = reinterpret_cast<const char*>(a.mo + qrow * D);
#pragma unroll
        for (int off = 0; off < D * 2; off += 128) prefetch_l2(m0 + off);
      }
    }
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

  // ------------------------------------------------------------- setup
  if (warp == 5) {
    tmem_alloc(tmem_slot, kOwnTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(&bars[oQFull], 1);
    for (int q = 0; q < kSt; ++q) {
      mbar_init(&bars[oKFull0 + q], 1);
      mbar_init(&bars[oKEmpty0 + q], 1);
      mbar_init(&bars[oVFull0 + q], 1);
      mbar_init(&bars[oVEmpty0 + q], 1);
    }
    mbar_init(&bars[oSFull], 1);
    mbar_init(&bars[oPFull], kRows);
    mbar_init(&bars[oOFull], 1);
    mbar_init(&bars[oDone], 1);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;

  if (warp < 4) {
    // ========================================================= softmax warps
    const int r = tid;  // row = TMEM lane
    int64_t qrow = -1;  // this row's (token, head) row of Q, O and LSE
    if (r < nrows) qrow = (int64_t)(q0 + r) * g.Hq + h;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const uint32_t tS = tmem + lane_off + kOwnColS;
    const uint32_t tP = tS + kColP;
    const uint32_t tO = tmem + lane_off + kOwnColO;
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
      // one partial row at a time (its D/8 16-byte loads in flight together), so the row
      // and the TMEM slice fit the register budget of two CTAs per SM
      for (int q = 0; q < npmax || q == 0; ++q) {  // warp-uniform: TMEM access is per warp
        const bool have = q < np;
        const float w = have ? ex2(__ldg(folded ? a.mlse + qrow : a.part_lse + pbase + q) * kLog2e - m) : 0.f;
        const __half* srow = !have ? a.part_o : (folded ? a.mo + qrow * D : a.part_o + (pbase + q) * D);
        const uint4* src = reinterpret_cast<const uint4*>(srow);
        uint4 hv[D / 8];
#pragma unroll
        for (int c = 0; c < D / 8; ++c) hv[c] = have ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        l += w;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          if (q > 0) {
            tmem_ld32(tO + c * 32, o);
            tmem_wait_ld();
          } else {
#pragma unroll
            for (int x = 0; x < 32; ++x) o[x] = 0u;
          }
          const __half2* hp = reinterpret_cast<const __half2*>(&hv[c * 4]);
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float2 f = __half22float2(hp[x]);
            o[2 * x] = __float_as_uint(fmaf(w, f.x, __uint_as_float(o[2 * x])));
            o[2 * x + 1] = __float_as_uint(fmaf(w, f.y, __uint_as_float(o[2 * x + 1])));
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
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[oSFull], j & 1, g.err));
      if (!ok) break;
      tc_fence_after();
      // scaled-logit row max (log2 units) from a first read of S; the causal mask applies to
      // the diagonal chunk only.  S is read from TMEM again, 64 columns at a time, for the
      // exponentials: half a row in registers at a time fits two CTAs per SM.
      bool masked = j == diag;
      int lim = masked ? r + 1 : kBN;
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
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t sr[2][32];
        tmem_ld32(tS + (2 * hf) * 32, sr[0]);
        tmem_ld32(tS + (2 * hf + 1) * 32, sr[1]);
        tmem_wait_ld();
        if (!masked) {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int x = 0; x < 32; x += 2)
              mv[(x >> 1) & 7] = max3(mv[(x >> 1) & 7], __uint_as_float(sr[c][x]), __uint_as_float(sr[c][x + 1]));
        } else {
#pragma unroll
          for (int c = 0; c < 2; ++c)
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if ((2 * hf + c) * 32 + x < lim) mv[x & 7] = fmaxf(mv[x & 7], __uint_as_float(sr[c][x]));
        }
      }
      float mx = fmaxf(fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3])), fmaxf(fmaxf(mv[4], mv[5]), fmaxf(mv[6], mv[7])));
      mx *= c2;
      // running max: rescale the TMEM accumulator only when it grows by more than 2^8
      // (p <= 256 otherwise, harmless in fp32 sums and bf16 P).  At this point the previous
      // PV has completed: the MMA that produced this S was issued after it.
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
      // p = 2^(s*c2 - m); P (bf16 pairs) overwrites the first 64 S columns: columns 0..63
      // are read before P's first 32 columns are written, 64..127 are never overwritten.
      // Unmasked chunks work on pairs with f32x2 arithmetic and send a share of the
      // exponentials to the FMA pipe; the diagonal chunk keeps the plain scalar form.
      float rv[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) rv[q] = 0.f;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t sr[2][32];
        tmem_ld32(tS + (2 * cc) * 32, sr[0]);
        tmem_ld32(tS + (2 * cc + 1) * 32, sr[1]);
        tmem_wait_ld();
        uint32_t pk[32];
        if (!masked) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const int pi = x >> 1;
              float u0, u1, p0, p1;
              fma2(u0, u1, __uint_as_float(sr[h2][x]), __uint_as_float(sr[h2][x + 1]), c2, c2, -m, -m);
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
              float p0 = ex2(fmaf(__uint_as_float(sr[h2][x]), c2, -m));
              float p1 = ex2(fmaf(__uint_as_float(sr[h2][x + 1]), c2, -m));
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
      mbar_arrive(&bars[oPFull]);
    }
    // ------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars[oOFull], 0, g.err));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / l;
      const float lse_row = (m + __log2f(l)) * kLn2;
      // The final O row (bf16) and LSE.  Each thread stages its own row in the Q and K
      // buffers (free: the O barrier implies every MMA completed; rows padded by 16 bytes so
      // the row-per-thread 16-byte writes spread over the banks) and hands it to the TMA
      // engine as one bulk copy.  The copies drain to memory on their own; the thread only
      // waits until the engine has read the staged row.
      constexpr int kStgBytes = D * 2 + 16;
      static_assert(4 * 32 * kStgBytes <= L::kV0, "staging rows");
      uint8_t* srow = smem + L::kQ + r * kStgBytes;
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
  } else if (warp == 4) {
    // ========================================================= TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(&bars[oQFull], L::kTile);
#pragma unroll
      for (int hh = 0; hh < D / 64; ++hh)
        tma_load_3d(smem + L::kQ + hh * kRows * 128, &tmQ, &bars[oQFull], hh * 64, h, q0);
      for (int j = 0; j < nchunks && ok; ++j) {
        const int st = j % kSt, u = j / kSt;
        const int tok = key0 + j * kBN;
        if (u > 0) ok = mbar_wait(&bars[oKEmpty0 + st], (u - 1) & 1, g.err);
        if (!ok) break;
        mbar_expect_tx(&bars[oKFull0 + st], L::kTile);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(smem + L::kK0 + st * L::kTile + hh * kRows * 128, &tmK, &bars[oKFull0 + st], hh * 64, gk, tok);
        if (u > 0) ok = mbar_wait(&bars[oVEmpty0 + st], (u - 1) & 1, g.err);
        if (!ok) break;
        mbar_expect_tx(&bars[oVFull0 + st], L::kTile);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh)
          tma_load_3d(smem + L::kV0 + st * L::kTile + hh * kRows * 128, &tmV, &bars[oVFull0 + st], hh * 64, gk, tok);
      }
    }
  } else {
    // ========================================================= MMA issuer (whole warp, one elected lane issues)
    constexpr uint32_t idS = idesc_bf16(kRows, kBN, false, false);
    constexpr uint32_t idO = idesc_bf16(kRows, D, false, true);
    const uint32_t sQ = smem_u32(smem + L::kQ);
    const uint32_t sK0 = smem_u32(smem + L::kK0);
    const uint32_t sV0 = smem_u32(smem + L::kV0);
    auto issue_s = [&](int j) {
      const uint32_t kb = sK0 + (j % kSt) * L::kTile;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
        mma_bf16_ss_warp(tmem + kOwnColS, sdesc_sw128(sQ + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024), idS,
                         kk > 0 ? 1u : 0u);
      }
      mma_commit_warp(&bars[oSFull]);
      mma_commit_warp(&bars[oKEmpty0 + j % kSt]);
    };
    auto issue_pv = [&](int j) {
      const uint32_t vb = sV0 + (j % kSt) * L::kTile;
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        mma_bf16_ts_warp(tmem + kOwnColO, tmem + kOwnColS + kColP + kk * 8,
                         sdesc_sw128(vb + kk * 2048, kRows * 128, 1024), idO, 1u);  // O starts from the merge
      mma_commit_warp(&bars[oVEmpty0 + j % kSt]);
    };
    ok = mbar_wait_warp(&bars[oQFull], 0, g.err) && mbar_wait_warp(&bars[oKFull0], 0, g.err);
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
    for (int j = 0; j < nchunks && ok; ++j) {
      ok = mbar_wait_warp(&bars[oVFull0 + j % kSt], (j / kSt) & 1, g.err) && mbar_wait_warp(&bars[oPFull], j & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_pv(j);  // reads P(j) before the next S overwrites it: one issuer, in-order MMAs
      if (j + 1 == nchunks) {
        mma_commit_warp(&bars[oOFull]);
        break;
      }
      ok = mbar_wait_warp(&bars[oKFull0 + (j + 1) % kSt], ((j + 1) / kSt) & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_s(j + 1);
    }
    mma_commit_warp(&bars[oDone]);
    mbar_wait_warp(&bars[oDone], 0, g.err);
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, kOwnTmemCols);
  }
}

template <int D, bool kNaive>
cudaError_t launch_tiles(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                         const int32_t* sel, const Work& w, __nv_bfloat16* O, float* LSE, int premerged,
                         cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e = make_rows_map(&tk, K, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tq, Q, (uint64_t)g.T, g.Hq, D, kRows);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tv, V, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  AttnArgs a{g, Q, sel, w.tile_off, w.tile_bucket, w.rows, w.part_o, w.part_lse, O, LSE, premerged,
             w.merged_o, w.merged_lse};
  const int smem = OwnLayout<D>::kAlloc;
  e = cudaFuncSetAttribute(attn_own_kernel<D, kNaive>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t items = (int64_t)g.num_seqs * g.MB * (g.bs / kRows) * g.Hq;
  if (items <= 0) return cudaSuccess;
  if (items > INT32_MAX) return cudaErrorInvalidConfiguration;
  attn_own_kernel<D, kNaive><<<(unsigned)items, kOwnThreads, smem, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_own_tiles(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                             const int32_t* sel, const Work& w, __nv_bfloat16* O, float* LSE, int premerged,
                             cudaStream_t st) {
  if (g.D == 64) return launch_tiles<64, false>(g, Q, K, V, sel, w, O, LSE, premerged, st);
  return launch_tiles<128, false>(g, Q, K, V, sel, w, O, LSE, premerged, st);
}

cudaError_t launch_naive_tiles(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                               const __nv_bfloat16* V, const int32_t* sel, __nv_bfloat16* O, float* LSE,
                               cudaStream_t st) {
  Work w{};
  if (g.D == 64) return launch_tiles<64, true>(g, Q, K, V, sel, w, O, LSE, 0, st);
  return launch_tiles<128, true>(g, Q, K, V, sel, w, O, LSE, 0, st);
}

}  // namespace moba
