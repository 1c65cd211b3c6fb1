// Block mean-pooling of the keys: Kbar[s, b, g, :] = mean of K over block b's valid tokens.
//
// The keys of one block of one sequence are a contiguous [n, Hkv*D] bf16 slab of K
// (n <= bs tokens, every KV head side by side), so one CTA reduces one slab: each
// thread owns a 16-byte column vector (8 bf16) and walks a strided subset of the
// rows, then the row groups are combined in a fixed order (deterministic).  HBM
// bound: K is read exactly once.  (youleyou.com, "Kimi发布MoBA突破性实现无限上下文",
// section "MoBA：基于块的混合注意力机制": a block is represented by the mean of its keys.)
#include "moba_internal.cuh"

namespace moba {

constexpr int kPoolThreads = 512;

__global__ void __launch_bounds__(kPoolThreads) pool_kernel(Geom g, const __nv_bfloat16* __restrict__ K,
                                                          float* __restrict__ Kbar) {
  extern __shared__ float red[];  // [rgroups, C]
  const int b = blockIdx.x, s = blockIdx.y;
  const int C = g.Hkv * g.D;
  const int nvec = C >> 3;
  const int32_t ts = seq_start(g, s);
  const int32_t te = seq_end(g, s);
  const int32_t t0 = ts + b * g.bs;
  const int32_t t1 = min(t0 + g.bs, te);
  const int n = t1 - t0;  // <= 0 for blocks past the sequence's end
  float* out = Kbar + ((size_t)s * g.MB + b) * (size_t)C;
  const int rg = nvec >= kPoolThreads ? 1 : kPoolThreads / nvec;  // row groups
  const int pairs = rg * nvec;
  for (int q = threadIdx.x; q < pairs; q += kPoolThreads) {
    const int r = q / nvec, v = q - r * nvec;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    const uint4* src = reinterpret_cast<const uint4*>(K + (size_t)t0 * C) + v;
    int t = r;
    for (; t + 3 * rg < n; t += 4 * rg) {
      uint4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = __ldg(src + (size_t)(t + u * rg) * nvec);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x[u]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float2 f = __bfloat1622float2(h[e]);
          acc[2 * e] += f.x;
          acc[2 * e + 1] += f.y;
        }
      }
    }
    for (; t < n; t += rg) {
      uint4 x = __ldg(src + (size_t)t * nvec);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float2 f = __bfloat1622float2(h[e]);
        acc[2 * e] += f.x;
        acc[2 * e + 1] += f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[r * C + v * 8 + e] = acc[e];
  }
  __syncthreads();
  const float inv = n > 0 ? 1.f / (float)n : 0.f;
  for (int c = threadIdx.x; c < C; c += kPoolThreads) {
    float sum = 0.f;
    for (int r = 0; r < rg; ++r) sum += red[r * C + c];
    out[c] = sum * inv;
  }
}

cudaError_t launch_pool(const Geom& g, const __nv_bfloat16* K, float* Kbar, cudaStream_t st) {
  const int C = g.Hkv * g.D;
  const int nvec = C >> 3;
  const int rg = nvec >= kPoolThreads ? 1 : kPoolThreads / nvec;
  const size_t smem = (size_t)rg * C * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(pool_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(g.MB, g.num_seqs);
  pool_kernel<<<grid, kPoolThreads, smem, st>>>(g, K, Kbar);
  return cudaGetLastError();
}

}  // namespace moba
