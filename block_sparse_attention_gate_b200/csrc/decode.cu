// Gated MoBA decode: one new query per sequence against its KV cache.
//
// The new token is the last token of its sequence (position p = len - 1, block i = p / bs),
// so it is gated exactly like a prefill row: the pooled keys of the earlier blocks b < i are
// scored by <q, Kbar[b]>, the own (possibly partial) block is always taken, and the best
// top_k - 1 earlier blocks join it (ties to the lower block index); attention runs over the
// selected blocks' keys only (the own block up to p) and the per-block results are merged
// by online softmax.  (MoBA README: "Parameter-less Gating Mechanism" and the FAQ answers of
// GitHub issue #27 on the forced current block; its FAQ answer of issue #30 notes that the
// released decode path skips the gate and runs full attention, which this one does not.)
//
// Decode is bound by HBM: one query row per (sequence, head) reads whole key blocks.  The
// kernels are therefore plain SIMT kernels built around coalesced row loads:
//   decode_gate_kernel : one CTA per (sequence, KV head); the group's pooled keys are staged
//                        in shared memory by 64-block chunks and one warp per query head
//                        scores them, keeping per-lane top lists merged at the end.
//   decode_attn_kernel : one CTA per (sequence, query head, selected block): eight warps
//                        take rounds of 32 keys; a round loads 32 K rows coalesced (a lane
//                        holds D/32 dimensions of each), forms the 32 dot products by a
//                        butterfly reduce-scatter (lane j ends with key j's logit), runs
//                        the online softmax, and accumulates P V with the lane again
//                        holding D/32 dimensions.  The CTA's eight partial states are
//                        combined into one normalised partial O and its LSE.
//   decode_merge_kernel: the top_k partials of a (sequence, head) merged by online softmax
//                        into the final O (bf16) and LSE.
#include <float.h>

#include "moba_internal.cuh"

namespace moba {

namespace {

constexpr int kGateChunk = 64;     // pooled-key rows staged per step of the gate
constexpr int kGateWarps = 8;      // query heads scored at once per CTA
constexpr int kAttnWarps = 8;
constexpr float kLog2eD = 1.4426950408889634f;
constexpr float kLn2D = 0.6931471805599453f;

__device__ __forceinline__ bool ranks_before(float sa, int32_t ba, float sb, int32_t bb) {
  return sa > sb || (sa == sb && ba < bb);
}

template <int D, int kMaxM>
__global__ void __launch_bounds__(kGateWarps * 32)
    decode_gate_kernel(Geom g, const __nv_bfloat16* __restrict__ Q, const float* __restrict__ Kbar,
                       int32_t* __restrict__ sel) {
  __shared__ float kb[kGateChunk][D + 1];   // +1: a lane's row walk hits a new bank each row
  __shared__ float qs[kGateWarps][D];
  const int s = blockIdx.y, gk = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t len = seq_end(g, s) - seq_start(g, s);
  const int i = (len - 1) / g.bs;          // own block (len >= 1: checked on the host)
  const int m = min(g.k - 1, i);
  const int64_t kb_row0 = (int64_t)s * g.MB;
  for (int h0 = 0; h0 < g.G; h0 += kGateWarps) {
    const int hh = h0 + warp;
    const bool live = hh < g.G;
    const int h = gk * g.G + hh;
    if (live)
      for (int d = lane; d < D; d += 32) qs[warp][d] = __bfloat162float(Q[((int64_t)s * g.Hq + h) * D + d]);
    // per-lane running top list (best first; ties to the lower index)
    float ls[kMaxM];
    int32_t lb[kMaxM];
#pragma unroll
    for (int q = 0; q < kMaxM; ++q) { ls[q] = -INFINITY; lb[q] = INT32_MAX; }
    for (int c0 = 0; c0 < i; c0 += kGateChunk) {
      const int n = min(kGateChunk, i - c0);
      __syncthreads();  // previous chunk consumed (and qs written)
      for (int e = threadIdx.x; e < n * D; e += kGateWarps * 32) {
        const int r = e / D, d = e - r * D;
        kb[r][d] = __ldg(Kbar + ((kb_row0 + c0 + r) * g.Hkv + gk) * D + d);
      }
      __syncthreads();
      if (live) {
#pragma unroll
        for (int u = 0; u < kGateChunk / 32; ++u) {
          const int r = u * 32 + lane;
          if (r < n) {
            float acc = 0.f;
#pragma unroll 16
            for (int d = 0; d < D; ++d) acc = fmaf(qs[warp][d], kb[r][d], acc);
            const int32_t b = c0 + r;
            // candidates reach a lane in ascending index: a new one goes after every listed
            // entry whose score is >= its own
            bool ge[kMaxM];
#pragma unroll
            for (int q = 0; q < kMaxM; ++q) ge[q] = ls[q] >= acc;
#pragma unroll
            for (int q = kMaxM - 1; q >= 1; --q) {
              ls[q] = ge[q] ? ls[q] : (ge[q - 1] ? acc : ls[q - 1]);
              lb[q] = ge[q] ? lb[q] : (ge[q - 1] ? b : lb[q - 1]);
            }
            ls[0] = ge[0] ? ls[0] : acc;
            lb[0] = ge[0] ? lb[0] : b;
          }
        }
      }
    }
    if (live) {
      int32_t* out = sel + ((int64_t)s * g.Hq + h) * g.k;
      if (lane == 0) out[0] = i;
      // m rounds of a warp-wide arg-best over the lanes' list heads; the winner pops its head
      for (int q = 0; q < m; ++q) {
        float bs_ = ls[0];
        int32_t bb = lb[0];
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) {
          const float os = __shfl_xor_sync(0xffffffffu, bs_, off);
          const int32_t ob = __shfl_xor_sync(0xffffffffu, bb, off);
          if (ranks_before(os, ob, bs_, bb)) { bs_ = os; bb = ob; }
        }
        if (lane == 0) out[1 + q] = bb;
        if (lb[0] == bb) {
#pragma unroll
          for (int x = 0; x + 1 < kMaxM; ++x) { ls[x] = ls[x + 1]; lb[x] = lb[x + 1]; }
          ls[kMaxM - 1] = -INFINITY;
          lb[kMaxM - 1] = INT32_MAX;
        }
      }
      for (int q = 1 + m + lane; q < g.k; q += 32) out[q] = -1;
    }
  }
}

// One (sequence, query head, selected block): normalised partial O (fp32) and its LSE.
template <int D>
__global__ void __launch_bounds__(kAttnWarps * 32)
    decode_attn_kernel(Geom g, const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ K,
                       const __nv_bfloat16* __restrict__ V, const int32_t* __restrict__ sel,
                       float* __restrict__ part_o, float* __restrict__ part_lse) {
  constexpr int kDL = D / 32;  // dimensions per lane
  __shared__ float red_m[kAttnWarps], red_l[kAttnWarps];
  __shared__ float red_o[kAttnWarps][D];
  const int slot = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = ((int64_t)s * g.Hq + h) * g.k + slot;
  const int32_t b = __ldg(sel + unit);
  if (b < 0) return;  // unused slot: the merge skips it
  const int32_t ts = seq_start(g, s);
  const int32_t len = seq_end(g, s) - ts;
  const int32_t p = len - 1;
  const int i = p / g.bs;
  const int32_t t0 = ts + b * g.bs;
  const int n = b == i ? p - b * g.bs + 1 : g.bs;  // own block: keys up to the new token
  const int gk = h / g.G;
  // this lane's query dimensions, pre-scaled into log2 units
  float q[kDL];
  {
    const __nv_bfloat16* qp = Q + ((int64_t)s * g.Hq + h) * D + lane * kDL;
#pragma unroll
    for (int x = 0; x < kDL; ++x) q[x] = __bfloat162float(qp[x]) * g.scale_log2;
  }
  const int64_t kv_stride = (int64_t)g.Hkv * D;
  const __nv_bfloat16* kbase = K + (int64_t)t0 * kv_stride + (int64_t)gk * D + lane * kDL;
  const __nv_bfloat16* vbase = V + (int64_t)t0 * kv_stride + (int64_t)gk * D + lane * kDL;
  float m = -INFINITY, l = 0.f;
  float o[kDL];
#pragma unroll
  for (int x = 0; x < kDL; ++x) o[x] = 0.f;
  for (int r0 = warp * 32; r0 < n; r0 += kAttnWarps * 32) {
    const int nk = min(32, n - r0);
    // partial dot products: v[j] = sum over this lane's dimensions of q . K[r0 + j]
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      float acc = 0.f;
      if (j < nk) {
        const __nv_bfloat16* kp = kbase + (int64_t)(r0 + j) * kv_stride;
        if constexpr (kDL == 4) {
          const uint2 raw = __ldg(reinterpret_cast<const uint2*>(kp));
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
          const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
          acc = fmaf(q[0], a.x, fmaf(q[1], a.y, fmaf(q[2], c.x, q[3] * c.y)));
        } else {
          const uint32_t raw = __ldg(reinterpret_cast<const uint32_t*>(kp));
          const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
          acc = fmaf(q[0], a.x, q[1] * a.y);
        }
      }
      v[j] = acc;
    }
    // butterfly reduce-scatter: after step `off` a lane keeps the half of the entries whose
    // index bit `off` equals its own lane bit; at the end lane j holds the sum for key j
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      const bool upper = (lane & off) != 0;
#pragma unroll
      for (int x = 0; x < off; ++x) {
        const float send = upper ? v[x] : v[x + off];
        const float keep = upper ? v[x + off] : v[x];
        v[x] = keep + __shfl_xor_sync(0xffffffffu, send, off);
      }
    }
    const float z = lane < nk ? v[0] : -INFINITY;  // logit of key r0 + lane, log2 units
    float mx = z;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    const float m_new = fmaxf(m, mx);
    const float alpha = exp2f(m - m_new);  // 0 on the first round (m = -inf)
    const float pz = lane < nk ? exp2f(z - m_new) : 0.f;
    float ps = pz;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
    l = l * alpha + ps;
    m = m_new;
#pragma unroll
    for (int x = 0; x < kDL; ++x) o[x] *= alpha;
    // the value rows of the round, eight at a time: the eight loads are in flight together
    // (a loop, not unrolled, so the registers stay few and several CTAs fit on an SM)
#pragma unroll 1
    for (int j0 = 0; j0 < 32; j0 += 8) {
      uint32_t vr[8][kDL / 2];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const __nv_bfloat16* vp = vbase + (int64_t)(r0 + j0 + j) * kv_stride;
        if constexpr (kDL == 4) {
          uint2 raw = make_uint2(0u, 0u);
          if (j0 + j < nk) raw = __ldg(reinterpret_cast<const uint2*>(vp));
          vr[j][0] = raw.x;
          vr[j][1] = raw.y;
        } else {
          vr[j][0] = j0 + j < nk ? __ldg(reinterpret_cast<const uint32_t*>(vp)) : 0u;
        }
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float pj = __shfl_sync(0xffffffffu, pz, j0 + j);  // 0 for keys past the block's end
#pragma unroll
        for (int x = 0; x < kDL / 2; ++x) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&vr[j][x]));
          o[2 * x] = fmaf(pj, f.x, o[2 * x]);
          o[2 * x + 1] = fmaf(pj, f.y, o[2 * x + 1]);
        }
      }
    }
  }
  // combine the warps' states (a warp with no keys has m = -inf, l = 0, o = 0)
  if (lane == 0) {
    red_m[warp] = m;
    red_l[warp] = l;
  }
#pragma unroll
  for (int x = 0; x < kDL; ++x) red_o[warp][lane * kDL + x] = o[x];
  __syncthreads();
  if (warp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, red_m[w]);
    float L = 0.f, acc[kDL];
#pragma unroll
    for (int x = 0; x < kDL; ++x) acc[x] = 0.f;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) {
      const float sc = red_l[w] > 0.f ? exp2f(red_m[w] - M) : 0.f;
      L += red_l[w] * sc;
#pragma unroll
      for (int x = 0; x < kDL; ++x) acc[x] = fmaf(red_o[w][lane * kDL + x], sc, acc[x]);
    }
    const float inv = 1.f / L;  // L >= 1: the maximum key contributes 2^0
#pragma unroll
    for (int x = 0; x < kDL; ++x) part_o[unit * D + lane * kDL + x] = acc[x] * inv;
    if (lane == 0) part_lse[unit] = (M + log2f(L)) * kLn2D;
  }
}

// The top_k partials of one (sequence, query head) merged by online softmax.
template <int D>
__global__ void __launch_bounds__(128)
    decode_merge_kernel(Geom g, const int32_t* __restrict__ sel, const float* __restrict__ part_o,
                        const float* __restrict__ part_lse, __nv_bfloat16* __restrict__ O,
                        float* __restrict__ LSE) {
  constexpr int kDL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * 4 + warp;  // (sequence, head)
  if (row >= (int64_t)g.num_seqs * g.Hq) return;
  float M = -INFINITY;
  for (int q = 0; q < g.k; ++q)
    if (__ldg(sel + row * g.k + q) >= 0) M = fmaxf(M, __ldg(part_lse + row * g.k + q) * kLog2eD);
  float L = 0.f, acc[kDL];
#pragma unroll
  for (int x = 0; x < kDL; ++x) acc[x] = 0.f;
  for (int q = 0; q < g.k; ++q) {
    if (__ldg(sel + row * g.k + q) < 0) continue;
    const float w = exp2f(__ldg(part_lse + row * g.k + q) * kLog2eD - M);
    L += w;
    const float* src = part_o + (row * g.k + q) * D + lane * kDL;
#pragma unroll
    for (int x = 0; x < kDL; ++x) acc[x] = fmaf(w, __ldg(src + x), acc[x]);
  }
  const float inv = 1.f / L;
#pragma unroll
  for (int x = 0; x < kDL; x += 2) {
    const __nv_bfloat162 b2 = __floats2bfloat162_rn(acc[x] * inv, acc[x + 1] * inv);
    *reinterpret_cast<__nv_bfloat162*>(O + row * D + lane * kDL + x) = b2;
  }
  if (lane == 0) LSE[row] = (M + log2f(L)) * kLn2D;
}

template <int D>
cudaError_t launch_decode_d(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                            const __nv_bfloat16* V, const float* Kbar, int32_t* sel, float* part_o,
                            float* part_lse, __nv_bfloat16* O, float* LSE, cudaStream_t st) {
  const dim3 ggrid((unsigned)g.Hkv, (unsigned)g.num_seqs);
  const int m = g.k - 1;
  if (m <= 2) decode_gate_kernel<D, 2><<<ggrid, kGateWarps * 32, 0, st>>>(g, Q, Kbar, sel);
  else if (m <= 4) decode_gate_kernel<D, 4><<<ggrid, kGateWarps * 32, 0, st>>>(g, Q, Kbar, sel);
  else if (m <= 8) decode_gate_kernel<D, 8><<<ggrid, kGateWarps * 32, 0, st>>>(g, Q, Kbar, sel);
  else decode_gate_kernel<D, kMaxTopK - 1><<<ggrid, kGateWarps * 32, 0, st>>>(g, Q, Kbar, sel);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  decode_attn_kernel<D><<<dim3((unsigned)g.k, (unsigned)g.Hq, (unsigned)g.num_seqs), kAttnWarps * 32, 0, st>>>(
      g, Q, K, V, sel, part_o, part_lse);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t rows = (int64_t)g.num_seqs * g.Hq;
  decode_merge_kernel<D><<<(unsigned)((rows + 3) / 4), 128, 0, st>>>(g, sel, part_o, part_lse, O, LSE);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                          const float* Kbar, int32_t* sel, float* part_o, float* part_lse, __nv_bfloat16* O,
                          float* LSE, cudaStream_t st) {
  if (g.D == 64) return launch_decode_d<64>(g, Q, K, V, Kbar, sel, part_o, part_lse, O, LSE, st);
  return launch_decode_d<128>(g, Q, K, V, Kbar, sel, part_o, part_lse, O, LSE, st);
}

}  // namespace moba
