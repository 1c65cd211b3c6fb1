// MoBA block attention, CUDA-core version: one warp per query row.
//
// Past blocks: every routed partial (token, query head, slot) attends the full block
// it selected (a past block is complete and wholly visible) and writes a normalised
// partial output and its log-sum-exp.  Own block: each (token, query head) attends its
// own block causally, then merges the past partials by online softmax and writes O and
// LSE.  (youleyou.com article, section "PyTorch实现关键要点": attention on the own
// block and on the selected blocks, merged by online softmax; zhuoshang.net
// "MoBA是什么？…", section "MoBA的技术原理": causal mask inside the current block.)
#include <float.h>

#include "moba_internal.cuh"

namespace moba {

constexpr int kSimtWarps = 8;
constexpr float kLn2 = 0.6931471805599453f;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum_bcast(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return __shfl_sync(0xffffffffu, v, 0);
}

// Online-softmax attention of one warp's query (q in shared memory, pre-scaled by
// scale*log2(e)) over keys [j0, j1) of KV head gk.  Returns the running max m (log2
// units), the sum l and the unnormalised accumulator (lane owns dims lane + 32*dd).
template <int D>
__device__ __forceinline__ void warp_attend(const Geom& g, const float* q, const __nv_bfloat16* __restrict__ K,
                                            const __nv_bfloat16* __restrict__ V, int gk, int32_t j0,
                                            int32_t j1, float& m, float& l, float (&acc)[D / 32]) {
  const int lane = threadIdx.x & 31;
  m = -INFINITY;
  l = 0.f;
#pragma unroll
  for (int dd = 0; dd < D / 32; ++dd) acc[dd] = 0.f;
  for (int32_t jc = j0; jc < j1; jc += 32) {
    const int32_t j = jc + lane;
    float sj = -INFINITY;
    if (j < j1) {
      const uint4* kr = reinterpret_cast<const uint4*>(K + ((size_t)j * g.Hkv + gk) * D);
      float dot = 0.f;
#pragma unroll
      for (int c = 0; c < D / 8; ++c) {
        uint4 x = __ldg(kr + c);
        const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(hx[e]);
          dot = fmaf(q[8 * c + 2 * e], f.x, dot);
          dot = fmaf(q[8 * c + 2 * e + 1], f.y, dot);
        }
      }
      sj = dot;
    }
    const float mn = fmaxf(m, warp_max(sj));
    const float alpha = exp2f(m - mn);
    const float pj = (j < j1) ? exp2f(sj - mn) : 0.f;
    l = l * alpha + warp_sum_bcast(pj);
#pragma unroll
    for (int dd = 0; dd < D / 32; ++dd) acc[dd] *= alpha;
    const int nk = min(32, j1 - jc);
    for (int kk = 0; kk < nk; ++kk) {
      const float pk = __shfl_sync(0xffffffffu, pj, kk);
      const __nv_bfloat16* vr = V + ((size_t)(jc + kk) * g.Hkv + gk) * D;
#pragma unroll
      for (int dd = 0; dd < D / 32; ++dd) acc[dd] = fmaf(pk, __bfloat162float(vr[lane + 32 * dd]), acc[dd]);
    }
    m = mn;
  }
}

template <int D>
__global__ void __launch_bounds__(kSimtWarps * 32) attn_past_simt_kernel(
    Geom g, const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ rows, float* __restrict__ part_o, float* __restrict__ part_lse) {
  __shared__ float qs[kSimtWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t pos = (int64_t)blockIdx.x * kSimtWarps + warp;
  const int32_t total = __ldg(offsets + g.nbk);
  if (pos >= total) return;
  // bucket holding this position: last bucket whose offset is <= pos
  int64_t lo = 0, hi = g.nbk - 1;
  while (lo < hi) {
    int64_t mid = (lo + hi + 1) >> 1;
    if (__ldg(offsets + mid) <= pos) lo = mid; else hi = mid - 1;
  }
  const int32_t b = (int32_t)(lo % g.MB);
  const int s = (int)((lo / g.MB) % g.num_seqs);
  const int gk = (int)(lo / ((int64_t)g.MB * g.num_seqs));
  const int32_t e = __ldg(rows + pos);
  const int64_t qrow = e / (g.k - 1);
  for (int d = lane; d < D; d += 32) qs[warp][d] = __bfloat162float(Q[qrow * D + d]) * g.scale_log2;
  __syncwarp();
  const int32_t j0 = seq_start(g, s) + b * g.bs;
  float m, l, acc[D / 32];
  warp_attend<D>(g, qs[warp], K, V, gk, j0, j0 + g.bs, m, l, acc);
  const float inv = 1.f / l;
#pragma unroll
  for (int dd = 0; dd < D / 32; ++dd) part_o[(size_t)e * D + lane + 32 * dd] = acc[dd] * inv;
  if (lane == 0) part_lse[e] = (m + log2f(l)) * kLn2;
}

template <int D>
__global__ void __launch_bounds__(kSimtWarps * 32) attn_self_merge_simt_kernel(
    Geom g, const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
    const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ sel,
    const float* __restrict__ part_o, const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ O,
    float* __restrict__ LSE) {
  __shared__ float qs[kSimtWarps][D];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t qrow = (int64_t)blockIdx.x * kSimtWarps + warp;
  if (qrow >= (int64_t)g.T * g.Hq) return;
  const int32_t t = (int32_t)(qrow / g.Hq);
  const int h = (int)(qrow - (int64_t)t * g.Hq);
  const int s = find_seq(g, t);
  const int32_t ts = seq_start(g, s);
  const int32_t i = (t - ts) / g.bs;
  const int gk = h / g.G;
  for (int d = lane; d < D; d += 32) qs[warp][d] = __bfloat162float(Q[qrow * D + d]) * g.scale_log2;
  __syncwarp();
  float m, l, acc[D / 32];
  warp_attend<D>(g, qs[warp], K, V, gk, ts + i * g.bs, t + 1, m, l, acc);
  const float lse_self = (m + log2f(l)) * kLn2;
  float M = lse_self;
  for (int slot = 1; slot < g.k; ++slot) {
    const int32_t b = __ldg(sel + qrow * g.k + slot);
    if (b >= 0 && b < i) M = fmaxf(M, __ldg(part_lse + qrow * (g.k - 1) + slot - 1));
  }
  const float ws = expf(lse_self - M) / l;
  float sumw = expf(lse_self - M);
  float o[D / 32];
#pragma unroll
  for (int dd = 0; dd < D / 32; ++dd) o[dd] = acc[dd] * ws;
  for (int slot = 1; slot < g.k; ++slot) {
    const int32_t b = __ldg(sel + qrow * g.k + slot);
    if (b >= 0 && b < i) {
      const int64_t e = qrow * (g.k - 1) + slot - 1;
      const float w = expf(__ldg(part_lse + e) - M);
      sumw += w;
#pragma unroll
      for (int dd = 0; dd < D / 32; ++dd) o[dd] = fmaf(w, __ldg(part_o + e * D + lane + 32 * dd), o[dd]);
    }
  }
  const float inv = 1.f / sumw;
#pragma unroll
  for (int dd = 0; dd < D / 32; ++dd) O[qrow * D + lane + 32 * dd] = __float2bfloat16_rn(o[dd] * inv);
  if (lane == 0) LSE[qrow] = M + logf(sumw);
}

cudaError_t launch_attn_past(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const Work& w, cudaStream_t st) {
  if (g.T == 0 || g.k < 2 || g.R == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((g.R + kSimtWarps - 1) / kSimtWarps);
  if (g.D == 64)
    attn_past_simt_kernel<64><<<grid, kSimtWarps * 32, 0, st>>>(g, Q, K, V, w.offsets, w.rows, w.part_o, w.part_lse);
  else
    attn_past_simt_kernel<128><<<grid, kSimtWarps * 32, 0, st>>>(g, Q, K, V, w.offsets, w.rows, w.part_o, w.part_lse);
  return cudaGetLastError();
}

cudaError_t launch_attn_self(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const int32_t* sel, const Work& w,
                             __nv_bfloat16* O, float* LSE, cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  const int64_t rows = (int64_t)g.T * g.Hq;
  const unsigned grid = (unsigned)((rows + kSimtWarps - 1) / kSimtWarps);
  if (g.D == 64)
    attn_self_merge_simt_kernel<64><<<grid, kSimtWarps * 32, 0, st>>>(g, Q, K, V, sel, w.part_o, w.part_lse, O, LSE);
  else
    attn_self_merge_simt_kernel<128><<<grid, kSimtWarps * 32, 0, st>>>(g, Q, K, V, sel, w.part_o, w.part_lse, O, LSE);
  return cudaGetLastError();
}

int launches_per_forward(const Geom& g) {
  // pool + gate + (route count, scan, scatter + past attention when top_k > 1) + own block/merge
  return 2 + (g.k > 1 ? 4 : 0) + 1;
}

}  // namespace moba
