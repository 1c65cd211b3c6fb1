// Block mean-pooling of the keys: Kbar[s, b, g, :] = mean of K over block b's valid tokens.
//
// The keys of one block of one sequence form a contiguous [n, Hkv*D] bf16 slab of K (n <= bs
// tokens, every KV head side by side).  A CTA reduces a 64-column strip of one slab: its 8
// column vectors (16 bytes = 8 bf16 each, so every row segment is one 128-byte line) times
// 32 row groups; each thread accumulates every 32nd row in fp32 and the row groups are
// summed in a fixed order (deterministic).  HBM bound: K is read exactly once, by
// blocks x strips CTAs.  (youleyou.com, "Kimi发布MoBA突破性实现无限上下文", section
// "MoBA：基于块的混合注意力机制": a block is represented by the mean of its keys.)
#include "moba_internal.cuh"

namespace moba {

constexpr int kPoolThreads = 256;
constexpr int kStripVec = 8;                            // 16-byte vectors per strip row
constexpr int kStripCols = kStripVec * 8;               // 64 bf16 columns
constexpr int kRowGroups = kPoolThreads / kStripVec;    // 32

// last_only: grid.y is 1 and each sequence's last block (the one holding its newest token)
// is pooled, for keeping Kbar current while a KV cache grows token by token.
__global__ void __launch_bounds__(kPoolThreads) pool_kernel(Geom g, const __nv_bfloat16* __restrict__ K,
                                                          float* __restrict__ Kbar, int last_only) {
  __shared__ float red[kRowGroups][kStripCols + 1];
  const int strip = blockIdx.x, s = blockIdx.z;
  const int b = last_only ? max(0, (seq_end(g, s) - seq_start(g, s) - 1) / g.bs) : (int)blockIdx.y;
  const int C = g.Hkv * g.D;
  const int32_t t0 = seq_start(g, s) + b * g.bs;
  const int32_t t1 = min(t0 + g.bs, seq_end(g, s));
  const int n = t1 - t0;  // <= 0 for blocks past the sequence's end
  const int v = threadIdx.x % kStripVec, r = threadIdx.x / kStripVec;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.f;
  const int cvec = C >> 3;  // 16-byte vectors per token row
  const uint4* src = reinterpret_cast<const uint4*>(K) + (size_t)t0 * cvec + strip * kStripVec + v;
  int t = r;
  for (; t + 3 * kRowGroups < n; t += 4 * kRowGroups) {
    uint4 x[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) x[u] = __ldg(src + (size_t)(t + u * kRowGroups) * cvec);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(&x[u]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = __bfloat1622float2(hx[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
  }
  for (; t < n; t += kRowGroups) {
    const uint4 x = __ldg(src + (size_t)t * cvec);
    const __nv_bfloat162* hx = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(hx[e]);
      acc[2 * e] += f.x;
      acc[2 * e + 1] += f.y;
    }
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[r][v * 8 + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < kStripCols) {
    float sum = 0.f;
    for (int q = 0; q < kRowGroups; ++q) sum += red[q][threadIdx.x];
    const float inv = n > 0 ? 1.f / (float)n : 0.f;
    Kbar[((size_t)s * g.MB + b) * C + strip * kStripCols + threadIdx.x] = sum * inv;
  }
}

cudaError_t launch_pool(const Geom& g, const __nv_bfloat16* K, float* Kbar, cudaStream_t st) {
  const int C = g.Hkv * g.D;  // a multiple of 64 (D is 64 or 128)
  dim3 grid(C / kStripCols, g.MB, g.num_seqs);
  pool_kernel<<<grid, kPoolThreads, 0, st>>>(g, K, Kbar, 0);
  return cudaGetLastError();
}

cudaError_t launch_pool_last(const Geom& g, const __nv_bfloat16* K, float* Kbar, cudaStream_t st) {
  const int C = g.Hkv * g.D;
  dim3 grid(C / kStripCols, 1, g.num_seqs);
  pool_kernel<<<grid, kPoolThreads, 0, st>>>(g, K, Kbar, 1);
  return cudaGetLastError();
}

}  // namespace moba
