// MoBA past-block attention on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// A work item is two tiles of 128 routed query rows of one bucket (KV head g, sequence s,
// past block b): every row that chose block b, laid out tile by tile by the routing step.
// The item attends the whole block (bs keys; a past block is complete and fully visible)
// and writes each row's normalised partial O (fp16: its rounding, at most 2^-11 of |O|
// per element, is far below the bf16 rounding of the final output) and LSE (fp32) at the
// row's partial id, for the own-block kernel to merge.  (youleyou.com, "Kimi发布MoBA突破性实现
// 无限上下文", section "PyTorch实现关键要点": attention runs on the chosen blocks separately
// and the results are merged by online softmax.)
//
// Per 128-key chunk j of tile t: S_t = Q_t K_j^T (tcgen05 SS MMA, fp32 in TMEM); softmax of
// S_t in registers (one thread per row = TMEM lane), P_t (bf16) written back over the first
// half of S_t's TMEM columns; O_t += P_t V_j (tcgen05 TS MMA).  The tensor core works on one
// tile while the other tile's softmax runs.
#include <cudaTypedefs.h>
#include <float.h>

#include "attn_common.cuh"

namespace moba {

namespace {

// ===================================================================== persistent past mode
// One CTA per SM walks the tile pairs blockIdx.x, blockIdx.x + gridDim.x, ...  Barrier phases
// run on across items: K/V stages and the S/P barriers count chunks globally (J), the Q, O
// and O-drained barriers count items (n).  The next item's routed rows are read early and its
// Q gather goes out as soon as this item's last S of the tile has completed; its first S MMAs
// then overlap this item's epilogue.  The epilogue stages 8 rows per warp at a time in a
// dedicated region (the Q and K/V buffers already hold the next item's data).
enum PBar {
  pQFull = 0, pKFull0, pKFull1, pKEmpty0, pKEmpty1, pVFull0, pVFull1, pVEmpty0, pVEmpty1,
  pSFull0, pSFull1, pPFull0, pPFull1, pOFull0, pOFull1, pODrained0, pODrained1, pDone, pNumBars
};
template <int D>
struct PLayout {
  static constexpr int kTile = kRows * D * 2;
  static constexpr int kQ = 0;
  static constexpr int kK0 = kQ + 2 * kTile;
  static constexpr int kV0 = kK0 + 2 * kTile;
  static constexpr int kBar = kV0 + 2 * kTile;
  static constexpr int kStgRow = D * 2 + 16;  // fp16 row, padded by 16 bytes
  static constexpr int kStg = kBar + 256;     // 8 warps x 8 rows
  static constexpr int kBytes = kStg + 8 * 8 * kStgRow;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_past_persistent_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                                AttnArgs a) {
  using L = PLayout<D>;
  static_assert(pNumBars * 8 + 4 <= 256, "barrier area");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kBar + pNumBars * 8);
  const Geom& g = a.g;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int32_t total = __ldg(a.tile_off + g.nbk);
  const int32_t first = (int32_t)blockIdx.x, stride = (int32_t)gridDim.x;
  if (first >= total) return;
  const int nitems = (total - 1 - first) / stride + 1;
  const int nchunks = g.bs / kBN;

  // ------------------------------------------------------------- item 0's rows and Q gather
  int32_t e_cur = -1;
  auto gather_q = [&](int t, int r, int32_t e) {
    const int64_t qrow = e >= 0 ? e / (g.k - 1) : -1;
    const __nv_bfloat16* src = qrow >= 0 ? a.Q + qrow * D : a.Q;
    const uint32_t nb = qrow >= 0 ? 16u : 0u;
    const uint32_t sQ = smem_u32(smem + L::kQ + t * L::kTile);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) cp_async_16(sQ + sw128_offset(r, c, kRows), src + c * 8, nb);
  };
  if (warp < 8) {
    const int t = warp >> 2, r = tid & (kRows - 1);
    e_cur = __ldg(a.rows + (int64_t)first * kPastTileRows + t * kRows + r);
    gather_q(t, r, e_cur);
  }

  // ------------------------------------------------------------- setup
  if (warp == 9) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
    tc_fence_before();
  }
  if (tid == 0) {
    mbar_init(&bars[pQFull], 2 * kRows);
    for (int q = 0; q < 2; ++q) {
      mbar_init(&bars[pKFull0 + q], 1);
      mbar_init(&bars[pKEmpty0 + q], 1);
      mbar_init(&bars[pVFull0 + q], 1);
      mbar_init(&bars[pVEmpty0 + q], 1);
      mbar_init(&bars[pSFull0 + q], 1);
      mbar_init(&bars[pPFull0 + q], kRows);
      mbar_init(&bars[pOFull0 + q], 1);
      mbar_init(&bars[pODrained0 + q], kRows);
    }
    mbar_init(&bars[pDone], 1);
    fence_mbar_init();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  bool ok = true;
  if (warp >= 8) regs_dec<kOtherRegs>(); else regs_inc<kSoftmaxRegs>();

  if (warp < 8) {
    // ========================================================= softmax warpgroups
    const int t = warp >> 2;
    const int r = tid & (kRows - 1);
    const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + kColS + t * kBN;
    const uint32_t tP = tS + kColP;
    const uint32_t tO = tmem + lane_off + kColO + t * 128;
    const float c2 = g.scale_log2;
    cp_async_wait_all();
    fence_proxy_async_smem();
    mbar_arrive(&bars[pQFull]);
    uint32_t J = 0;
    for (int n = 0; n < nitems && ok; ++n) {
      const bool has_next = n + 1 < nitems;
      const int32_t e_next =
          has_next ? __ldg(a.rows + (int64_t)(first + (n + 1) * stride) * kPastTileRows + t * kRows + r) : -1;
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < nchunks && ok; ++j, ++J) {
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[pSFull0 + t], J & 1, g.err));
        if (!ok) break;
        tc_fence_after();
        uint32_t sr[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(tS + c * 32, sr[c]);
        tmem_wait_ld();
        if (j == nchunks - 1 && has_next) gather_q(t, r, e_next);  // Q_t is free: its last S completed
        float mv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) mv[q] = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c)
#pragma unroll
          for (int x = 0; x < 32; x += 2)
            mv[(x >> 1) & 7] = max3(mv[(x >> 1) & 7], __uint_as_float(sr[c][x]), __uint_as_float(sr[c][x + 1]));
        float mx = fmaxf(fmaxf(fmaxf(mv[0], mv[1]), fmaxf(mv[2], mv[3])), fmaxf(fmaxf(mv[4], mv[5]), fmaxf(mv[6], mv[7])));
        mx *= c2;
        if (j == 0) {
          m = mx;
        } else if (__any_sync(0xffffffffu, mx > m + kRescaleLog2)) {
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
        float rv[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) rv[q] = 0.f;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t pk[32];
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
          tmem_st32(tP + cc * 32, pk);
        }
        l += ((rv[0] + rv[1]) + (rv[2] + rv[3])) + ((rv[4] + rv[5]) + (rv[6] + rv[7]));
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bars[pPFull0 + t]);
      }
      if (!ok) break;
      if (has_next) {  // the next item's Q rows of this tile have landed
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(&bars[pQFull]);
      }
      // ------------------------------------------------------- epilogue of item n
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[pOFull0 + t], n & 1, g.err));
      if (!ok) break;
      tc_fence_after();
      const float inv_l = 1.f / l;
      const float lse_row = (m + __log2f(l)) * kLn2;
      uint32_t hv[D / 2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; x += 2) {
          const __half2 h2v = __floats2half2_rn(__uint_as_float(o[x]) * inv_l, __uint_as_float(o[x + 1]) * inv_l);
          hv[c * 16 + (x >> 1)] = *reinterpret_cast<const uint32_t*>(&h2v);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[pODrained0 + t]);  // O_t may now be overwritten by the next item
      if (e_cur >= 0) a.part_lse[e_cur] = lse_row;
      uint8_t* slot = smem + L::kStg + (warp * 8 + (lane & 7)) * L::kStgRow;
#pragma unroll
      for (int rnd = 0; rnd < 4; ++rnd) {
        if ((lane >> 3) == rnd) {
#pragma unroll
          for (int x = 0; x < D / 2; x += 4)
            *reinterpret_cast<uint4*>(slot + x * 4) = make_uint4(hv[x], hv[x + 1], hv[x + 2], hv[x + 3]);
          if (e_cur >= 0) {
            fence_proxy_async_smem();
            bulk_store_s2g(a.part_o + (int64_t)e_cur * D, smem_u32(slot), D * 2);
            bulk_commit();
            bulk_wait_read_all();
          }
        }
        __syncwarp();
      }
      e_cur = e_next;
    }
  } else if (warp == 8) {
    // ========================================================= TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      uint32_t J = 0;
      int64_t lo_next = __ldg(a.tile_bucket + first);
      for (int n = 0; n < nitems && ok; ++n) {
        const int64_t lo = lo_next;
        if (n + 1 < nitems) lo_next = __ldg(a.tile_bucket + first + (n + 1) * stride);
        const int32_t b = (int32_t)(lo % g.MB);
        const int s = (int)((lo / g.MB) % g.num_seqs);
        const int gk = (int)(lo / ((int64_t)g.MB * g.num_seqs));
        const int32_t key0 = seq_start(g, s) + b * g.bs;
        for (int j = 0; j < nchunks && ok; ++j, ++J) {
          const int st = J & 1;
          const uint32_t u = J >> 1;
          const int tok = key0 + j * kBN;
          if (u > 0) ok = mbar_wait(&bars[pKEmpty0 + st], (u - 1) & 1, g.err);
          if (!ok) break;
          mbar_expect_tx(&bars[pKFull0 + st], L::kTile);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d(smem + L::kK0 + st * L::kTile + hh * kRows * 128, &tmK, &bars[pKFull0 + st], hh * 64, gk, tok);
          if (u > 0) ok = mbar_wait(&bars[pVEmpty0 + st], (u - 1) & 1, g.err);
          if (!ok) break;
          mbar_expect_tx(&bars[pVFull0 + st], L::kTile);
#pragma unroll
          for (int hh = 0; hh < D / 64; ++hh)
            tma_load_3d(smem + L::kV0 + st * L::kTile + hh * kRows * 128, &tmV, &bars[pVFull0 + st], hh * 64, gk, tok);
        }
      }
    }
  } else if (warp == 9) {
    // ========================================================= MMA issuer (whole warp)
    constexpr uint32_t idS = idesc_bf16(kRows, kBN, false, false);
    constexpr uint32_t idO = idesc_bf16(kRows, D, false, true);
    const uint32_t sQ = smem_u32(smem + L::kQ);
    const uint32_t sK0 = smem_u32(smem + L::kK0);
    const uint32_t sV0 = smem_u32(smem + L::kV0);
    auto issue_s = [&](int t, uint32_t jj) {
      const uint32_t qb = sQ + t * L::kTile, kb = sK0 + (jj & 1) * L::kTile;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
        mma_ss_lo(tmem + kColS + t * kBN, sdesc_lo(qb + off, 16), sdesc_lo(kb + off, 16), idS, kk > 0 ? 1u : 0u);
      }
      mma_commit_warp(&bars[pSFull0 + t]);
    };
    auto issue_pv = [&](int t, uint32_t jj, bool first_chunk) {
      const uint32_t vb = sV0 + (jj & 1) * L::kTile;
#pragma unroll
      for (int kk = 0; kk < kBN / 16; ++kk)
        mma_ts_lo(tmem + kColO + t * 128, tmem + kColS + t * kBN + kColP + kk * 8, sdesc_lo(vb + kk * 2048, kRows * 128),
                  idO, (!first_chunk || kk > 0) ? 1u : 0u);
    };
    uint32_t J = 0;
    for (int n = 0; n < nitems && ok; ++n) {
      ok = mbar_wait_warp(&bars[pQFull], n & 1, g.err) && mbar_wait_warp(&bars[pKFull0 + (J & 1)], (J >> 1) & 1, g.err);
      if (!ok) break;
      tc_fence_after();
      issue_s(0, J);
      issue_s(1, J);
      mma_commit_warp(&bars[pKEmpty0 + (J & 1)]);
      for (int j = 0; j < nchunks && ok; ++j) {
        const uint32_t Jc = J + j;
        const bool more = j + 1 < nchunks;
        ok = mbar_wait_warp(&bars[pVFull0 + (Jc & 1)], (Jc >> 1) & 1, g.err) &&
             mbar_wait_warp(&bars[pPFull0], Jc & 1, g.err);
        if (ok && j == 0 && n > 0) ok = mbar_wait_warp(&bars[pODrained0], (n - 1) & 1, g.err);
        if (!ok) break;
        tc_fence_after();
        issue_pv(0, Jc, j == 0);
        if (!more) mma_commit_warp(&bars[pOFull0]);
        if (more) {
          ok = mbar_wait_warp(&bars[pKFull0 + ((Jc + 1) & 1)], ((Jc + 1) >> 1) & 1, g.err);
          if (!ok) break;
          tc_fence_after();
          issue_s(0, Jc + 1);
        }
        ok = mbar_wait_warp(&bars[pPFull1], Jc & 1, g.err);
        if (ok && j == 0 && n > 0) ok = mbar_wait_warp(&bars[pODrained1], (n - 1) & 1, g.err);
        if (!ok) break;
        tc_fence_after();
        issue_pv(1, Jc, j == 0);
        mma_commit_warp(&bars[pVEmpty0 + (Jc & 1)]);
        if (!more) mma_commit_warp(&bars[pOFull1]);
        if (more) {
          issue_s(1, Jc + 1);
          mma_commit_warp(&bars[pKEmpty0 + ((Jc + 1) & 1)]);
        }
      }
      J += nchunks;
    }
    mma_commit_warp(&bars[pDone]);
    mbar_wait_warp(&bars[pDone], 0, g.err);
  }

  // ------------------------------------------------------------- teardown
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int D>
cudaError_t launch_past_persistent(const Geom& g, const __nv_bfloat16* K, const __nv_bfloat16* V, const __nv_bfloat16* Q,
                                   const Work& w, cudaStream_t st) {
  CUtensorMap tk, tv;
  cudaError_t e = make_rows_map(&tk, K, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  e = make_rows_map(&tv, V, (uint64_t)g.T, g.Hkv, D, kBN);
  if (e != cudaSuccess) return e;
  AttnArgs a{g, Q, nullptr, w.tile_off, w.tile_bucket, w.rows, w.part_o, w.part_lse, nullptr, nullptr, 0,
             nullptr, nullptr};
  const int smem = PLayout<D>::kAlloc;
  e = cudaFuncSetAttribute(attn_past_persistent_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, attn_past_persistent_kernel<D>);
  if (e != cudaSuccess) return e;
  if ((uint32_t)fa.numRegs < kLaunchRegs) return cudaErrorInvalidConfiguration;
  int dev = 0, nsm = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = past_tiles(g);
  dim3 grid((unsigned)(tiles < nsm ? tiles : nsm));
  attn_past_persistent_kernel<D><<<grid, kThreads, smem, st>>>(tk, tv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_past(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const Work& w, cudaStream_t st) {
  if (g.T == 0 || g.k < 2 || g.R == 0) return cudaSuccess;
  if (g.D == 64) return launch_past_persistent<64>(g, K, V, Q, w, st);
  return launch_past_persistent<128>(g, K, V, Q, w, st);
}

}  // namespace moba
