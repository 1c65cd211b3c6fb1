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
//   decode_attn_tma_kernel: one CTA per (sequence, query head, selected block).  A producer
//                        warp streams the block's keys and values by TMA, 128 keys per
//                        stage, into a three-stage shared-memory ring; four consumer warps
//                        each form 32 logits per stage (a lane per key, the key row read
//                        from the swizzled stage, the query broadcast from shared memory),
//                        run the online softmax and accumulate P V (a lane per D/32
//                        dimensions).  The copies in flight, not the threads' registers,
//                        carry the memory parallelism.  The four warps' states are combined
//                        into one normalised partial O and its LSE.
//   decode_merge_kernel: the top_k partials of a (sequence, head) merged by online softmax
//                        into the final O (bf16) and LSE.
#include <cudaTypedefs.h>
#include <float.h>

#include "moba_internal.cuh"
#include "sm100.cuh"

namespace moba {

namespace {

constexpr int kGateChunk = 64;     // pooled-key rows staged per step of the gate
constexpr int kGateWarps = 8;      // query heads scored at once per CTA
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

// One (sequence, query head, selected block) per CTA, fed by TMA: warp 4 streams the
// block's keys and values, 128 keys per stage, into a three-stage shared-memory ring
// (three 64 KB stages in flight per SM: the copies, not the threads' registers, hold the
// memory parallelism), and warps 0-3 each take 32 keys of every stage.  A warp forms its
// 32 logits with a lane per key (the key row read from the 128-byte-swizzled stage, the
// query broadcast from shared memory), runs the online softmax over them, and accumulates
// P V with a lane per D/32 dimensions.  The four warps' states are combined at the end into
// the unit's normalised partial O and its LSE.
constexpr int kTKeys = 128;     // keys per stage
constexpr int kTStages = 3;
constexpr int kTConsumers = 4;  // consumer warps (32 keys of each stage each)

template <int D>
struct DLayout {
  static constexpr int kTile = kTKeys * D * 2;       // [128 x D] bf16
  static constexpr int kK0 = 0;                       // kTStages stages
  static constexpr int kV0 = kK0 + kTStages * kTile;  // kTStages stages
  static constexpr int kQ = kV0 + kTStages * kTile;   // [D] fp32, pre-scaled
  static constexpr int kRed = kQ + D * 4;             // [4][D] partial O + [4] m, l
  static constexpr int kBar = kRed + kTConsumers * D * 4 + 2 * kTConsumers * 4;
  static constexpr int kBytes = kBar + 64;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__((kTConsumers + 1) * 32, 1)
    decode_attn_tma_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                           Geom g, const __nv_bfloat16* __restrict__ Q, const int32_t* __restrict__ sel,
                           float* __restrict__ part_o, float* __restrict__ part_lse) {
  using L = DLayout<D>;
  constexpr int kDL = D / 32;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* empty = full + kTStages;
  float* qs = reinterpret_cast<float*>(smem + L::kQ);
  float* red_o = reinterpret_cast<float*>(smem + L::kRed);
  float* red_m = red_o + kTConsumers * D;
  float* red_l = red_m + kTConsumers;
  const int slot = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t unit = ((int64_t)s * g.Hq + h) * g.k + slot;
  const int32_t b = __ldg(sel + unit);
  if (b < 0) return;  // unused slot: the merge skips it
  const int32_t ts = seq_start(g, s);
  const int32_t p = seq_end(g, s) - ts - 1;
  const int i = p / g.bs;
  const int32_t t0 = ts + b * g.bs;
  const int n = b == i ? p - b * g.bs + 1 : g.bs;  // own block: keys up to the new token
  const int nch = (n + kTKeys - 1) / kTKeys;
  const int gk = h / g.G;
  if (threadIdx.x < D) qs[threadIdx.x] = __bfloat162float(Q[((int64_t)s * g.Hq + h) * D + threadIdx.x]) * g.scale_log2;
  if (threadIdx.x == 0) {
    for (int q = 0; q < kTStages; ++q) {
      mbar_init(&full[q], 1);
      mbar_init(&empty[q], kTConsumers);
    }
    fence_mbar_init();
  }
  __syncthreads();
  bool ok = true;
  if (warp == kTConsumers) {
    // ========================================================= TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      for (int c = 0; c < nch && ok; ++c) {
        const int st = c % kTStages, u = c / kTStages;
        if (u > 0) ok = mbar_wait(&empty[st], (u - 1) & 1, g.err);
        if (!ok) break;
        mbar_expect_tx(&full[st], 2 * L::kTile);
#pragma unroll
        for (int hh = 0; hh < D / 64; ++hh) {
          tma_load_3d(smem + L::kK0 + st * L::kTile + hh * kTKeys * 128, &tmK, &full[st], hh * 64, gk, t0 + c * kTKeys);
          tma_load_3d(smem + L::kV0 + st * L::kTile + hh * kTKeys * 128, &tmV, &full[st], hh * 64, gk, t0 + c * kTKeys);
        }
      }
    }
  } else {
    // ========================================================= consumers
    float m = -INFINITY, l = 0.f;
    float o[kDL];
#pragma unroll
    for (int x = 0; x < kDL; ++x) o[x] = 0.f;
    const int r = warp * 32 + lane;  // this lane's key row inside a stage (logits)
    for (int c = 0; c < nch && ok; ++c) {
      const int st = c % kTStages;
      ok = __all_sync(0xffffffffu, mbar_wait(&full[st], (c / kTStages) & 1, g.err));
      if (!ok) break;
      const uint8_t* kst = smem + L::kK0 + st * L::kTile;
      const uint8_t* vst = smem + L::kV0 + st * L::kTile;
      // logit of key (c * 128 + r), log2 units: the row's 16-byte chunks sit at
      // (chunk ^ (row & 7)) inside each 128-byte, 64-dimension atom
      float z = 0.f;
#pragma unroll
      for (int a = 0; a < D / 64; ++a)
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 kv = *reinterpret_cast<const uint4*>(kst + a * kTKeys * 128 + r * 128 + ((ch ^ (r & 7)) << 4));
          const float4 qa = *reinterpret_cast<const float4*>(qs + a * 64 + ch * 8);
          const float4 qb = *reinterpret_cast<const float4*>(qs + a * 64 + ch * 8 + 4);
          const float2 k0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kv.x));
          const float2 k1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kv.y));
          const float2 k2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kv.z));
          const float2 k3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kv.w));
          z = fmaf(qa.x, k0.x, fmaf(qa.y, k0.y, fmaf(qa.z, k1.x, fmaf(qa.w, k1.y, z))));
          z = fmaf(qb.x, k2.x, fmaf(qb.y, k2.y, fmaf(qb.z, k3.x, fmaf(qb.w, k3.y, z))));
        }
      const bool live = c * kTKeys + r < n;
      if (!live) z = -INFINITY;
      float mx = z;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m, mx);
      if (m_new != -INFINITY) {  // warp-uniform: some key of this warp's share is live
        const float alpha = exp2f(m - m_new);
        const float pz = live ? exp2f(z - m_new) : 0.f;
        float ps = pz;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l = l * alpha + ps;
        m = m_new;
#pragma unroll
        for (int x = 0; x < kDL; ++x) o[x] *= alpha;
        // P V: lane holds dimensions [kDL * lane, kDL * lane + kDL) of each value row
        const int d0 = kDL * lane;
        const int a = d0 >> 6, ch = (d0 & 63) >> 3, within = (d0 & 7) * 2;
#pragma unroll 8
        for (int j = 0; j < 32; ++j) {
          const float pj = __shfl_sync(0xffffffffu, pz, j);
          const int vr = warp * 32 + j;
          const uint8_t* vp = vst + a * kTKeys * 128 + vr * 128 + ((ch ^ (vr & 7)) << 4) + within;
          if constexpr (kDL == 4) {
            const uint2 raw = *reinterpret_cast<const uint2*>(vp);
            const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
            const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
            o[0] = fmaf(pj, f0.x, o[0]);
            o[1] = fmaf(pj, f0.y, o[1]);
            o[2] = fmaf(pj, f1.x, o[2]);
            o[3] = fmaf(pj, f1.y, o[3]);
          } else {
            const uint32_t raw = *reinterpret_cast<const uint32_t*>(vp);
            const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw));
            o[0] = fmaf(pj, f0.x, o[0]);
            o[1] = fmaf(pj, f0.y, o[1]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);  // this warp's share of the stage is read
    }
    // combine the four warps' states (a warp without live keys has m = -inf, l = 0, o = 0)
    if (lane == 0) {
      red_m[warp] = m;
      red_l[warp] = l;
    }
#pragma unroll
    for (int x = 0; x < kDL; ++x) red_o[warp * D + lane * kDL + x] = o[x];
  }
  __syncthreads();
  if (ok && warp == 0) {
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kTConsumers; ++w) M = fmaxf(M, red_m[w]);
    float Lsum = 0.f, acc[kDL];
#pragma unroll
    for (int x = 0; x < kDL; ++x) acc[x] = 0.f;
#pragma unroll
    for (int w = 0; w < kTConsumers; ++w) {
      const float sc = red_l[w] > 0.f ? exp2f(red_m[w] - M) : 0.f;
      Lsum += red_l[w] * sc;
#pragma unroll
      for (int x = 0; x < kDL; ++x) acc[x] = fmaf(red_o[w * D + lane * kDL + x], sc, acc[x]);
    }
    const float inv = 1.f / Lsum;  // >= 1: the largest key contributes 2^0
#pragma unroll
    for (int x = 0; x < kDL; ++x) part_o[unit * D + lane * kDL + x] = acc[x] * inv;
    if (lane == 0) part_lse[unit] = (M + log2f(Lsum)) * kLn2D;
  }
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
  {
    CUtensorMap tk, tv;
    if ((e = make_rows_map(&tk, K, (uint64_t)g.T, g.Hkv, D, kTKeys)) != cudaSuccess) return e;
    if ((e = make_rows_map(&tv, V, (uint64_t)g.T, g.Hkv, D, kTKeys)) != cudaSuccess) return e;
    const int smem = DLayout<D>::kAlloc;
    if ((e = cudaFuncSetAttribute(decode_attn_tma_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    decode_attn_tma_kernel<D><<<dim3((unsigned)g.k, (unsigned)g.Hq, (unsigned)g.num_seqs), (kTConsumers + 1) * 32,
                                smem, st>>>(tk, tv, g, Q, sel, part_o, part_lse);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
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
