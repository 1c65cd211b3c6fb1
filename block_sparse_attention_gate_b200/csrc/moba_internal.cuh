// Internal definitions shared by the MoBA kernels and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace moba {

constexpr int kMaxTopK = 16;
// Routed rows per past-block attention CTA (two 128-row tiles); route.cu tiles buckets by it.
constexpr int kPastTileRows = 256;

// Problem geometry as the kernels see it (passed by value).
struct Geom {
  const int32_t* cu;  // device offsets, or nullptr for uniform sequences of length L
  int32_t num_seqs;
  int32_t L;          // uniform sequence length (cu == nullptr)
  int32_t T;          // total tokens
  int32_t Hq, Hkv, G, D;
  int32_t bs;         // block size
  int32_t MB;         // max blocks per sequence
  int32_t k;          // top_k (own block included)
  float scale;        // softmax scale
  float scale_log2;   // softmax scale * log2(e)
  int64_t nbk;        // routing buckets: Hkv * num_seqs * MB
  int64_t R;          // routed partial rows: T * Hq * (k - 1)
  int* err;           // device error word (bounded waits that gave up), never null
};

// Rows with more than kPremergeMinPartials - 1 past partials (top_k - 1 >= 3) get them
// folded by a separate pass before the own-block kernel.
constexpr int kPremergeMinPartials = 3;
__host__ __device__ inline bool premerge_used(const Geom& g) {
  return g.T > 0 && g.k - 1 >= kPremergeMinPartials;
}

// Upper bound on the past-block attention tiles (kPastTileRows rows each): every bucket's
// last tile may be partial.
__host__ __device__ inline int64_t past_tiles(const Geom& g) {
  return (g.R + kPastTileRows - 1) / kPastTileRows + g.nbk;
}

__device__ __forceinline__ int32_t seq_start(const Geom& g, int s) {
  return g.cu ? __ldg(g.cu + s) : s * g.L;
}
__device__ __forceinline__ int32_t seq_end(const Geom& g, int s) {
  return g.cu ? __ldg(g.cu + s + 1) : (s + 1) * g.L;
}
// Sequence holding token t (binary search over the offsets).
__device__ __forceinline__ int find_seq(const Geom& g, int32_t t) {
  if (!g.cu) return t / g.L;
  int lo = 0, hi = g.num_seqs - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(g.cu + mid) <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Workspace carve-up (device pointers; every region 256-byte aligned).
struct Work {
  int32_t* counts;    // [nbk] rows routed to each (kv head, sequence, block) bucket
  int32_t* cursors;   // [nbk] scatter cursors
  int32_t* tile_off;  // [nbk + 1] exclusive scan of per-bucket tile counts
  int32_t* tile_bucket;  // [past_tiles(g)] bucket of each past-attention tile
  int32_t* rows;      // [past_tiles(g) * kPastTileRows] routed partial ids, tile by tile (-1: empty)
  __half* part_o;     // [R, D] normalised partial outputs (fp16)
  float* part_lse;    // [R] partial log-sum-exp
  __half* merged_o;   // [T * Hq, D] folded partials (only when premerge_used)
  float* merged_lse;  // [T * Hq]
  float* kbar;        // [num_seqs, MB, Hkv, D] (used by moba_fwd when the caller passes none)
  __nv_bfloat16* kbar_hi;  // [num_seqs, MB, Hkv, D] bf16 rn(Kbar) for the tensor-core gate
  __nv_bfloat16* kbar_lo;  // [num_seqs, MB, Hkv, D] bf16 rn(Kbar - hi)
  float* kbar_n2;     // [num_seqs, Hkv, MB] squared norms of the pooled keys (gate score bound)
  int32_t* sel;       // [T, Hq, k] (used by moba_fwd when the caller passes none)
  size_t bytes;       // total
};

// Launchers (each returns the launch's cudaError_t).
cudaError_t make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, int heads, int D, int box_rows);
cudaError_t launch_pool(const Geom& g, const __nv_bfloat16* K, float* Kbar, cudaStream_t st);
// Pools only each sequence's last block (the one holding its newest token).
cudaError_t launch_pool_last(const Geom& g, const __nv_bfloat16* K, float* Kbar, cudaStream_t st);
// Gated decode: gate, split-KV attention over the selected blocks, merge.  part_o
// [num_seqs * Hq * k, D] fp32 and part_lse [num_seqs * Hq * k] are scratch.
cudaError_t launch_decode(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                          const float* Kbar, int32_t* sel, float* part_o, float* part_lse, __nv_bfloat16* O,
                          float* LSE, cudaStream_t st);
cudaError_t launch_gate(const Geom& g, const __nv_bfloat16* Q, const float* Kbar, int32_t* sel,
                        const Work& w, cudaStream_t st);
cudaError_t launch_route(const Geom& g, const int32_t* sel, const Work& w, cudaStream_t st);
cudaError_t launch_attn_past(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const Work& w, cudaStream_t st);
cudaError_t launch_attn_self(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const int32_t* sel, const Work& w,
                             __nv_bfloat16* O, float* LSE, cudaStream_t st);
// Own-block attention + merge (attn_own.cu): one 128-token tile of one head per CTA; rows
// with two or more past partials read them folded from w.merged_* when premerged is set.
cudaError_t launch_own_tiles(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const int32_t* sel, const Work& w,
                             __nv_bfloat16* O, float* LSE, int premerged, cudaStream_t st);
cudaError_t launch_naive_tiles(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                               const __nv_bfloat16* V, const int32_t* sel, __nv_bfloat16* O, float* LSE,
                               cudaStream_t st);
// Mask-based form: every causal key scored, keys outside the selected blocks masked.
cudaError_t launch_attn_naive(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                              const __nv_bfloat16* V, const int32_t* sel, __nv_bfloat16* O, float* LSE,
                              cudaStream_t st);
// Backward through the selected blocks (selection held fixed): Dp pre-pass, routing, dQ
// partials of the routed slots, own block + final dQ, dK/dV.  Dp [T * Hq] and dq_part
// [R, D] fp32 are scratch; w carries the routing arrays.
cudaError_t launch_attn_bwd(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K, const __nv_bfloat16* V,
                            const __nv_bfloat16* O, const float* LSE, const __nv_bfloat16* dO, const int32_t* sel,
                            const Work& w, float* Dp, float* dq_part, __nv_bfloat16* dQ, __nv_bfloat16* dK,
                            __nv_bfloat16* dV, cudaStream_t st);
// Number of kernel launches one forward pass enqueues (pool, gate, route, attention).
int launches_per_forward(const Geom& g);

}  // namespace moba
