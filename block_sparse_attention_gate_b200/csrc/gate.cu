// Parameter-free MoBA gate: scores <q, Kbar[b]> over the strictly earlier blocks of the
// query's sequence, forced own block, top-(k-1) past blocks by descending score with
// ties to the lower block index.  (MoBA README, "Parameter-less Gating Mechanism" and the
// FAQ answer of GitHub issue #27; youleyou.com article, section "PyTorch实现关键要点".)
//
// One warp per (token, query head).  Lane j scores candidates b = j, j+32, ... in fp32
// (bf16 query times fp32 pooled key) and keeps a sorted private top list; the warp then
// merges the 32 lists with an exact (score desc, index asc) tournament.
#include <float.h>

#include "moba_internal.cuh"

namespace moba {

constexpr int kGateWarps = 8;

struct Cand {
  float s;
  int32_t b;
};

// a ranks before b: larger score, or equal score and lower block index
__device__ __forceinline__ bool ranks_before(float sa, int32_t ba, float sb, int32_t bb) {
  return sa > sb || (sa == sb && ba < bb);
}

__global__ void __launch_bounds__(kGateWarps * 32) gate_simt_kernel(Geom g, const __nv_bfloat16* __restrict__ Q,
                                                                  const float* __restrict__ Kbar,
                                                                  int32_t* __restrict__ sel) {
  extern __shared__ float qs[];  // [kGateWarps, D]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kGateWarps + warp;  // t * Hq + h
  if (row >= (int64_t)g.T * g.Hq) return;
  const int32_t t = (int32_t)(row / g.Hq);
  const int h = (int)(row - (int64_t)t * g.Hq);
  const int s = find_seq(g, t);
  const int32_t p = t - seq_start(g, s);
  const int32_t i = p / g.bs;
  const int gk = h / g.G;
  float* q = qs + warp * g.D;
  for (int d = lane; d < g.D; d += 32) q[d] = __bfloat162float(Q[row * g.D + d]);
  __syncwarp();
  const int m = min(g.k - 1, i);
  Cand top[kMaxTopK];
  int cnt = 0;
  const float* kb0 = Kbar + (((size_t)s * g.MB) * g.Hkv + gk) * (size_t)g.D;
  const size_t bstride = (size_t)g.Hkv * g.D;
  for (int32_t b = lane; b < i && m > 0; b += 32) {
    const float4* kb = reinterpret_cast<const float4*>(kb0 + (size_t)b * bstride);
    float acc = 0.f;
    for (int d4 = 0; d4 < (g.D >> 2); ++d4) {
      float4 v = __ldg(kb + d4);
      acc = fmaf(q[4 * d4 + 0], v.x, acc);
      acc = fmaf(q[4 * d4 + 1], v.y, acc);
      acc = fmaf(q[4 * d4 + 2], v.z, acc);
      acc = fmaf(q[4 * d4 + 3], v.w, acc);
    }
    // insert into the lane's sorted list (candidates arrive in ascending b)
    if (cnt < m || acc > top[m - 1].s) {
      int pos = cnt < m ? cnt : m - 1;
      while (pos > 0 && top[pos - 1].s < acc) {
        top[pos] = top[pos - 1];
        --pos;
      }
      top[pos].s = acc;
      top[pos].b = b;
      if (cnt < m) ++cnt;
    }
  }
  int32_t* out = sel + row * g.k;
  if (lane == 0) out[0] = i;
  int ptr = 0;
  for (int slot = 0; slot < m; ++slot) {
    float bs_ = ptr < cnt ? top[ptr].s : -FLT_MAX;
    int32_t bb = ptr < cnt ? top[ptr].b : INT32_MAX;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      float os = __shfl_xor_sync(0xffffffffu, bs_, off);
      int32_t ob = __shfl_xor_sync(0xffffffffu, bb, off);
      if (ranks_before(os, ob, bs_, bb)) {
        bs_ = os;
        bb = ob;
      }
    }
    if (ptr < cnt && top[ptr].b == bb) ++ptr;
    if (lane == 0) out[1 + slot] = bb;
  }
  for (int slot = 1 + m + lane; slot < g.k; slot += 32) out[slot] = -1;
}

cudaError_t launch_gate(const Geom& g, const __nv_bfloat16* Q, const float* Kbar, int32_t* sel,
                        const Work& w, cudaStream_t st) {
  (void)w;
  const int64_t rows = (int64_t)g.T * g.Hq;
  if (rows == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((rows + kGateWarps - 1) / kGateWarps);
  gate_simt_kernel<<<grid, kGateWarps * 32, kGateWarps * g.D * sizeof(float), st>>>(g, Q, Kbar, sel);
  return cudaGetLastError();
}

}  // namespace moba
