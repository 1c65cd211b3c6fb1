// MoBA block attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Two modes share one kernel body:
//   past : a CTA takes two tiles of 128 routed query rows of one bucket (KV head g,
//          sequence s, past block b), attends the whole block (bs keys; a past block is
//          complete and fully visible) and writes normalised partials (fp16) + LSE (fp32).
//   own  : a CTA takes two tiles of 128 tokens (two heads, or two consecutive tiles of one
//          head) inside one block.  Each row's past partials are merged FIRST: they become
//          the starting state (m, l, O) of the online softmax, which then runs over the
//          block's keys up to the diagonal (causal mask on the diagonal chunk) and ends with
//          the final O (bf16) and LSE.
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

#include "moba_internal.cuh"
#include "sm100.cuh"

namespace moba {

namespace {

constexpr int kThreads = 384;  // warps 0-3 softmax tile 0, 4-7 softmax tile 1, 8 TMA, 9 MMA, 10-11 idle
// Register split (setmaxnreg): the kernel is compiled for kLaunchRegs per thread; the third
// warpgroup gives registers back so the two softmax warpgroups can hold a full S row.
// 2 * 128 * kSoftmaxRegs + 128 * kOtherRegs must not exceed 384 * kLaunchRegs (checked on
// the host against the compiled register count before every launch).
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 216;
constexpr uint32_t kOtherRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= 384 * kLaunchRegs, "register split too large");
constexpr int kRows = 128;     // query rows per tile (M); two tiles per CTA
constexpr int kBN = 128;       // keys per chunk (N of S, K of PV)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // S of tile t at kColS + 128 t
constexpr uint32_t kColP = 0;      // P of tile t (bf16 pairs) aliased at S + 0 .. S + 63
constexpr uint32_t kColO = 256;    // O of tile t at kColO + 128 t
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;  // rescale O only when a row max grows by more than 2^8

// 2^x for a pair on the FMA pipe, for a share of the exponentials that would otherwise all
// queue on the MUFU unit: x = j + f with j = rint(x) (the 1.5 * 2^23 rounding trick) and
// f in [-0.5, 0.5]; 2^f from a degree-3 polynomial (relative error 7.5e-5; coefficients from
// our own iteratively reweighted least-squares fit of 2^f on that interval), 2^j added into
// the exponent field.  x is clamped to >= -126 so the exponent never wraps; below 2^-24 the
// result only has to be negligible next to the row sum, as it is.
constexpr int kPolyNum = 1, kPolyDen = 4;  // pairs (pair index mod kPolyDen) < kPolyNum use it
__device__ __forceinline__ void exp2_poly2(float& p0, float& p1, float x0, float x1) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0, t1, r0, r1, f0, f1, q0, q1;
  add2(t0, t1, x0, x1, kRound, kRound);
  add2(r0, r1, t0, t1, -kRound, -kRound);
  fma2(f0, f1, r0, r1, -1.f, -1.f, x0, x1);
  fma2(q0, q1, f0, f1, 0.05517132207751274f, 0.05517132207751274f, 0.24261054396629333f, 0.24261054396629333f);
  fma2(q0, q1, q0, q1, f0, f1, 0.6932609677314758f, 0.6932609677314758f);
  fma2(q0, q1, q0, q1, f0, f1, 0.9999281167984009f, 0.9999281167984009f);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

struct AttnArgs {
  Geom g;
  const __nv_bfloat16* Q;
  const int32_t* sel;
  const int32_t* tile_off;
  const int32_t* tile_bucket;
  const int32_t* rows;
  __half* part_o;
  float* part_lse;
  __nv_bfloat16* O;
  float* LSE;
  int own_head_pairs;  // own mode: tiles are heads (2p, 2p+1) of one group (else query tiles 2p, 2p+1)
};

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
  int64_t qrow_base;  // own mode: Q row of token q0 (t * Hq + h) ...
  int32_t q0;         // own mode: first token
  int h;              // own mode: query head
  int nrows;          // valid rows (0..128)
  int diag;           // own mode: index of the diagonal chunk
  int32_t row_start;  // past mode: first routed position
};

template <int D, bool kOwn>
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

  // ------------------------------------------------------------- work item
  int gk, s, i_blk = 0, nchunks;
  int32_t key0;
  TileInfo ti[2];
  if constexpr (!kOwn) {
    // The routed rows are laid out tile by tile (kPastTileRows slots per tile, -1 in the
    // slots past a bucket's last row), so a tile needs only its bucket and its own slots.
    const int32_t tile = (int32_t)blockIdx.x;
    const int32_t total = __ldg(a.tile_off + g.nbk);
    const int64_t lo = __ldg(a.tile_bucket + tile);  // in bounds for every launched tile
    if (tile >= total) return;
    const int32_t b = (int32_t)(lo % g.MB);
    s = (int)((lo / g.MB) % g.num_seqs);
    gk = (int)(lo / ((int64_t)g.MB * g.num_seqs));
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      ti[t].row_start = tile * kPastTileRows + t * kRows;
      ti[t].nrows = kRows;  // empty slots hold -1
      ti[t].diag = 1 << 30;
      ti[t].qrow_base = 0; ti[t].q0 = 0; ti[t].h = 0;
    }
    key0 = seq_start(g, s) + b * g.bs;
    nchunks = g.bs / kBN;
  } else {
    const int per_blk = g.bs / kRows;
    s = blockIdx.y;
    const int32_t ts = seq_start(g, s), te = seq_end(g, s);
    if (a.own_head_pairs) {
      i_blk = blockIdx.x / per_blk;
      const int qt = blockIdx.x - i_blk * per_blk;
      const int32_t q0 = ts + i_blk * g.bs + qt * kRows;
      if (q0 >= te) return;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        ti[t].h = 2 * blockIdx.z + t;
        ti[t].q0 = q0;
        ti[t].nrows = min(kRows, te - q0);
        ti[t].diag = qt;
        ti[t].row_start = 0;
      }
      nchunks = qt + 1;
    } else {
      const int pairs = (per_blk + 1) / 2;
      i_blk = blockIdx.x / pairs;
      const int qp = blockIdx.x - i_blk * pairs;
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
        ti[t].row_start = 0;
      }
      nchunks = has1 ? qt1 + 1 : 2 * qp + 1;
    }
    gk = ti[0].h / g.G;
    key0 = ts + i_blk * g.bs;
  }

  // ------------------------------------------------------------- early loads
  // Past mode: the softmax threads look up their routed rows and start the Q gather before
  // the setup below.
  int32_t e = -1;  // past mode: this thread's partial id (-1: empty slot)
  if (!kOwn && warp < 8) {
    const int t = warp >> 2, r = tid & (kRows - 1);
    {
      e = __ldg(a.rows + ti[t].row_start + r);
      const int64_t qrow = e >= 0 ? e / (g.k - 1) : -1;
      const __nv_bfloat16* src = qrow >= 0 ? a.Q + qrow * D : a.Q;
      const uint32_t nb = qrow >= 0 ? 16u : 0u;  // zeros for empty slots
      const uint32_t sQ = smem_u32(smem + L::kQ + t * L::kTile);
#pragma unroll
      for (int c = 0; c < D / 8; ++c) cp_async_16(sQ + sw128_offset(r, c, kRows), src + c * 8, nb);
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
    mbar_init(&bars[kQFull], kOwn ? 1 : 2 * kRows);  // own: one TMA transaction; past: every row's gather
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
    int64_t qrow = -1;  // own mode: this row's (token, head) row of Q, O and LSE
    if (kOwn && r < T_.nrows) qrow = (int64_t)(T_.q0 + r) * g.Hq + T_.h;
    if constexpr (!kOwn) {  // this row's Q gather (issued before the setup) has landed
      cp_async_wait_all();
      fence_proxy_async_smem();
      mbar_arrive(&bars[kQFull]);
    }
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS + t * kBN;
    const uint32_t tP = tS + kColP;
    const uint32_t tO = tmem + lane_off + kColO + t * 128;
    const float c2 = g.scale_log2;
    float m = -INFINITY, l = 0.f;
    if constexpr (kOwn) {
      // Merge first: the row's past partials (normalised O_q and LSE_q, written by the
      // past-block attention before this kernel runs) become the starting state of the
      // online softmax, in its log2 units: m = max_q LSE_q log2(e), w_q = 2^(LSE_q log2(e) - m),
      // l = sum_q w_q, O = sum_q w_q O_q (the past keys' share of sum_k 2^(s_k c2 - m) v_k).
      // The own block's chunks then continue the same online softmax; the O accumulator is
      // written here, before the first PV MMA (which accumulates onto it).
      int np = 0;
      int32_t pe[kMaxTopK - 1];
      float pl[kMaxTopK - 1];
      if (qrow >= 0) {
        int32_t bsel[kMaxTopK - 1];
#pragma unroll
        for (int q = 0; q < kMaxTopK - 1; ++q) bsel[q] = q + 1 < g.k ? __ldg(a.sel + qrow * g.k + q + 1) : -1;
#pragma unroll
        for (int q = 0; q < kMaxTopK - 1; ++q)
          if (bsel[q] >= 0 && bsel[q] < i_blk) pe[np++] = (int32_t)(qrow * (g.k - 1) + q);
#pragma unroll
        for (int q = 0; q < kMaxTopK - 1; ++q)
          if (q < np) pl[q] = __ldg(a.part_lse + pe[q]) * kLog2e;
      }
      for (int q = 0; q < np; ++q) m = fmaxf(m, pl[q]);
      const int npmax = __reduce_max_sync(0xffffffffu, np);
      for (int q0 = 0; q0 < npmax || q0 == 0; q0 += 2) {  // warp-uniform: TMEM access is per warp
        uint4 hv[2][D / 8];
        float w[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int q = q0 + h2;
          const bool have = q < np;
          w[h2] = have ? ex2(pl[q] - m) : 0.f;
          const uint4* src = reinterpret_cast<const uint4*>(a.part_o + (int64_t)(have ? pe[q] : 0) * D);
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
      const bool masked = kOwn && j >= T_.diag;
      const int lim = (kOwn && j == T_.diag) ? r + 1 : (masked ? 0 : kBN);
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
      if (!kOwn && j == 0) {
        m = mx;
      } else if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {  // own mode: m may start at -inf
        const float m_new = fmaxf(m, mx);
        const float alpha = ex2(m - m_new);
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
      // Past mode: the normalised partial row (fp16: its rounding, at most 2^-11 of |O| per
      // element, is far below the bf16 rounding of the final output) and its LSE, at the
      // row's partial id.  Own mode: the final O row (bf16) and LSE: the past partials were
      // merged in at the start.
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
          if constexpr (kOwn) {
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(v0, v1);
            hv[x >> 1] = *reinterpret_cast<const uint32_t*>(&b2);
          } else {
            const __half2 h2v = __floats2half2_rn(v0, v1);
            hv[x >> 1] = *reinterpret_cast<const uint32_t*>(&h2v);
          }
        }
#pragma unroll
        for (int x = 0; x < 16; x += 4)
          *reinterpret_cast<uint4*>(srow + c * 64 + x * 4) = make_uint4(hv[x], hv[x + 1], hv[x + 2], hv[x + 3]);
      }
      void* dst = nullptr;
      if constexpr (kOwn) {
        if (qrow >= 0) {
          a.LSE[qrow] = lse_row;
          dst = a.O + qrow * D;
        }
      } else {
        if (e >= 0) {
          a.part_lse[e] = lse_row;
          dst = a.part_o + (int64_t)e * D;
        }
      }
      if (dst) {
        fence_proxy_async_smem();
        bulk_store_s2g(dst, smem_u32(srow), D * 2);
        bulk_commit();
        bulk_wait_read_all();
      }
    }
  } else if (warp == 8) {
    // ========================================================= TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      if constexpr (kOwn) {  // both Q tiles: 128 consecutive tokens of one head each
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
                         sdesc_sw128(vb + kk * 2048, kRows * 128, 1024), idO, (kOwn || j > 0 || kk > 0) ? 1u : 0u);
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

template <int D, bool kOwn>
cudaError_t launch_tc(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                      const int32_t* sel, const Work& w, __nv_bfloat16* O, float* LSE, dim3 grid, int head_pairs,
                      cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  cudaError_t e = make_rows_map(&tk, K, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  if (kOwn) {
    e = make_rows_map(&tq, Q, (uint64_t)g.T, g.Hq, D, kRows);
    if (e != cudaSuccess) return e;
  } else {
    tq = tk;  // unused: past mode gathers its Q rows
  }
  e = make_rows_map(&tv, V, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  AttnArgs a{g, Q, sel, w.tile_off, w.tile_bucket, w.rows, w.part_o, w.part_lse, O, LSE, head_pairs};
  const int smem = Layout<D>::kAlloc;
  e = cudaFuncSetAttribute(attn_tc_kernel<D, kOwn>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // the setmaxnreg split must fit in what the launch reserves, or the increase never returns
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_tc_kernel<D, kOwn>);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
  attn_tc_kernel<D, kOwn><<<grid, kThreads, smem, st>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_past(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const Work& w, cudaStream_t st) {
  if (g.T == 0 || g.k < 2 || g.R == 0) return cudaSuccess;
  const int64_t tiles = past_tiles(g);  // bound on routed tile pairs
  dim3 grid((unsigned)tiles);
  if (g.D == 64) return launch_tc<64, false>(g, Q, K, V, nullptr, w, nullptr, nullptr, grid, 0, st);
  return launch_tc<128, false>(g, Q, K, V, nullptr, w, nullptr, nullptr, grid, 0, st);
}

cudaError_t launch_attn_self(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const int32_t* sel, const Work& w,
                             __nv_bfloat16* O, float* LSE, cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  const int per_blk = g.bs / kRows;
  const int head_pairs = (g.G % 2 == 0) ? 1 : 0;
  dim3 grid = head_pairs ? dim3((unsigned)(g.MB * per_blk), (unsigned)g.num_seqs, (unsigned)(g.Hq / 2))
                         : dim3((unsigned)(g.MB * ((per_blk + 1) / 2)), (unsigned)g.num_seqs, (unsigned)g.Hq);
  if (g.D == 64) return launch_tc<64, true>(g, Q, K, V, sel, w, O, LSE, grid, head_pairs, st);
  return launch_tc<128, true>(g, Q, K, V, sel, w, O, LSE, grid, head_pairs, st);
}

int launches_per_forward(const Geom& g) {
  // pool + gate (Kbar split, scores/top-k) + (route count, scan, scatter + past attention
  // when top_k > 1) + own block/merge
  return 3 + (g.k > 1 ? 4 : 0) + 1;
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
