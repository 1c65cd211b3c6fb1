// Query-to-block routing (the "organise the data" step of the youleyou.com article,
// section "PyTorch实现关键要点", done MoE-style): every (token, query head, slot >= 1)
// whose selected past block is b joins bucket (kv head g, sequence s, block b).
// Three passes: per-CTA shared-memory histograms flushed to global counts; a one-CTA
// exclusive scan of the attention tiles per bucket; scatter of partial ids.  The routed
// rows are laid out tile by tile: bucket b owns slots [tile_off[b], tile_off[b+1]) * tile_m,
// its rows first and -1 in the rest, so an attention tile reads only its own slots.
//
// A partial id is e = (t * Hq + h) * (k - 1) + (slot - 1); it indexes the partial
// output buffers directly, so the order inside a bucket does not affect any result.
#include "moba_internal.cuh"

namespace moba {

constexpr int kRouteThreads = 256;
constexpr int kScanThreads = 1024;

__device__ __forceinline__ int64_t bucket_of(const Geom& g, int gk, int s, int32_t b) {
  return ((int64_t)gk * g.num_seqs + s) * g.MB + b;
}

// grid (MB, num_seqs, Hkv): CTA = query block i of sequence s, KV head g
// The scatter pass also fills, for bucket (g, s, i - 1), the tile -> bucket table and the
// empty slots of its last tile (CTA (i, s, g) exists for every bucket that can hold rows, so
// each such bucket is covered exactly once).
template <bool kScatter>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(Geom g, const int32_t* __restrict__ sel,
                                                            int32_t* __restrict__ counts,
                                                            int32_t* __restrict__ cursors,
                                                            int32_t* __restrict__ rows,
                                                            const int32_t* __restrict__ tile_off,
                                                            int32_t* __restrict__ tile_bucket) {
  extern __shared__ int32_t hist[];  // [i] counts, then [i] bases (scatter)
  const int i = blockIdx.x, s = blockIdx.y, gk = blockIdx.z;
  const int32_t ts = seq_start(g, s), te = seq_end(g, s);
  const int32_t t0 = ts + i * g.bs;
  const int32_t n = min(t0 + g.bs, te) - t0;
  if (n <= 0 || i == 0 || g.k < 2) return;
  const int km1 = g.k - 1;
  int32_t* base = hist + i;
  for (int b = threadIdx.x; b < i; b += kRouteThreads) hist[b] = 0;
  __syncthreads();
  const int per_tok = g.G * km1;
  const int64_t nent = (int64_t)n * per_tok;
  for (int64_t e = threadIdx.x; e < nent; e += kRouteThreads) {
    const int32_t tl = (int32_t)(e / per_tok);
    const int rem = (int)(e - (int64_t)tl * per_tok);
    const int hh = rem / km1, slot = 1 + rem - hh * km1;
    const int h = gk * g.G + hh;
    const int32_t b = __ldg(sel + ((int64_t)(t0 + tl) * g.Hq + h) * g.k + slot);
    if (b >= 0 && b < i) atomicAdd(&hist[b], 1);
  }
  __syncthreads();
  if constexpr (!kScatter) {
    for (int b = threadIdx.x; b < i; b += kRouteThreads)
      if (hist[b]) atomicAdd(counts + bucket_of(g, gk, s, b), hist[b]);
  } else {
  {
    const int64_t bk = bucket_of(g, gk, s, i - 1);
    const int32_t t0 = __ldg(tile_off + bk), t1 = __ldg(tile_off + bk + 1);
    for (int32_t tt = t0 + threadIdx.x; tt < t1; tt += kRouteThreads) tile_bucket[tt] = (int32_t)bk;
    const int64_t slot_end = (int64_t)t1 * kPastTileRows;
    for (int64_t sl = (int64_t)t0 * kPastTileRows + __ldg(counts + bk) + threadIdx.x; sl < slot_end; sl += kRouteThreads)
      rows[sl] = -1;
  }
  for (int b = threadIdx.x; b < i; b += kRouteThreads) {
    const int c = hist[b];
    base[b] = c ? atomicAdd(cursors + bucket_of(g, gk, s, b), c) : 0;
    hist[b] = 0;
  }
  __syncthreads();
  for (int64_t e = threadIdx.x; e < nent; e += kRouteThreads) {
    const int32_t tl = (int32_t)(e / per_tok);
    const int rem = (int)(e - (int64_t)tl * per_tok);
    const int hh = rem / km1, slot = 1 + rem - hh * km1;
    const int h = gk * g.G + hh;
    const int64_t qrow = (int64_t)(t0 + tl) * g.Hq + h;
    const int32_t b = __ldg(sel + qrow * g.k + slot);
    if (b >= 0 && b < i) {
      const int32_t pos = base[b] + atomicAdd(&hist[b], 1);
      rows[pos] = (int32_t)(qrow * km1 + (slot - 1));
    }
  }
  }
}

// Exclusive scan of the bucket tile counts (tile = tile_m rows); each bucket's scatter
// cursor starts at its first slot.
__global__ void __launch_bounds__(kScanThreads) route_scan_kernel(int64_t nbk, int tile_m,
                                                                const int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ cursors,
                                                                int32_t* __restrict__ tile_off) {
  __shared__ int64_t st[kScanThreads];
  const int tid = threadIdx.x;
  const int64_t per = (nbk + kScanThreads - 1) / kScanThreads;
  const int64_t lo = min(nbk, per * tid), hi = min(nbk, lo + per);
  int64_t tl = 0;
  for (int64_t j = lo; j < hi; ++j) tl += (counts[j] + tile_m - 1) / tile_m;
  st[tid] = tl;
  __syncthreads();
  for (int off = 1; off < kScanThreads; off <<= 1) {
    const int64_t b = tid >= off ? st[tid - off] : 0;
    __syncthreads();
    st[tid] += b;
    __syncthreads();
  }
  int64_t tt = st[tid] - tl;
  for (int64_t j = lo; j < hi; ++j) {
    cursors[j] = (int32_t)(tt * tile_m);
    tile_off[j] = (int32_t)tt;
    tt += (counts[j] + tile_m - 1) / tile_m;
  }
  if (tid == kScanThreads - 1) tile_off[nbk] = (int32_t)st[tid];
}

cudaError_t launch_route_tiles(const Geom& g, const int32_t* sel, const Work& w, int tile_m,
                               cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * (size_t)g.nbk, st);
  if (e != cudaSuccess) return e;
  const size_t smem = 2 * sizeof(int32_t) * (size_t)g.MB;
  e = cudaFuncSetAttribute(route_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(route_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(g.MB, g.num_seqs, g.Hkv);
  route_kernel<false><<<grid, kRouteThreads, smem, st>>>(g, sel, w.counts, w.cursors, w.rows, w.tile_off, w.tile_bucket);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_scan_kernel<<<1, kScanThreads, 0, st>>>(g.nbk, tile_m, w.counts, w.cursors, w.tile_off);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  route_kernel<true><<<grid, kRouteThreads, smem, st>>>(g, sel, w.counts, w.cursors, w.rows, w.tile_off, w.tile_bucket);
  return cudaGetLastError();
}

cudaError_t launch_route(const Geom& g, const int32_t* sel, const Work& w, cudaStream_t st) {
  return launch_route_tiles(g, sel, w, kPastTileRows, st);
}

}  // namespace moba
