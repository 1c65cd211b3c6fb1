// Attention stage entry points of the own block (the pre-merge of a row's past partials,
// then the one-tile own-block kernel in attn_own.cu), the mask-based form, and the TMA
// tensor maps shared by the attention kernels.  (The past blocks are in attn_past.cu.)
#include <cudaTypedefs.h>
#include <float.h>

#include "attn_common.cuh"

namespace moba {

namespace {
// When a row can have more than two past partials, they are folded before the own-block
// kernel runs: one warp per (token, head) row with two or more partials loads all of them
// at once (a lane holds D/32 elements of each, so every partial row is one coalesced read),
// merges them by online softmax (M = max LSE_q, w_q = e^(LSE_q - M), O = sum w_q O_q /
// sum w_q, LSE = M + ln sum w_q) and writes the result to the row's entry of mo / mlse.
// The own-block kernel then merges one partial per row: a single round trip instead of one
// per two partials.  The partials themselves are left as they are.

template <int D>
__global__ void __launch_bounds__(256) premerge_kernel(Geom g, const int32_t* __restrict__ sel,
                                                       const __half* __restrict__ part_o,
                                                       const float* __restrict__ part_lse, __half* __restrict__ mo,
                                                       float* __restrict__ mlse) {
  constexpr int kDL = D / 32;  // elements of a partial row per lane
  const int lane = threadIdx.x & 31;
  const int64_t rows = (int64_t)g.T * g.Hq;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int km1 = g.k - 1;
  for (int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); row < rows; row += nwarps) {
    const int32_t t = (int32_t)(row / g.Hq);
    const int s = find_seq(g, t);
    const int i = (t - seq_start(g, s)) / g.bs;
    const int64_t base = row * km1;
    // One round trip per row: lane q reads slot q's block and LSE, and every lane reads its
    // share of all km1 partial rows at once (in bounds whether or not a slot is used; the
    // unused ones are excluded by a select below, never multiplied in).
    const int32_t b = lane < km1 ? __ldg(sel + row * g.k + 1 + lane) : -1;
    const float lq = lane < km1 ? __ldg(part_lse + base + lane) : -INFINITY;
    uint32_t raw[kMaxTopK - 1][kDL / 2];
#pragma unroll
    for (int q = 0; q < kMaxTopK - 1; ++q) {
      const __half* src = part_o + (base + (q < km1 ? q : 0)) * D + lane * kDL;
      if constexpr (kDL == 4) {
        const uint2 v = q < km1 ? __ldg(reinterpret_cast<const uint2*>(src)) : make_uint2(0u, 0u);
        raw[q][0] = v.x;
        raw[q][1] = v.y;
      } else {
        raw[q][0] = q < km1 ? __ldg(reinterpret_cast<const uint32_t*>(src)) : 0u;
      }
    }
    // the chosen past blocks fill the first np slots
    const uint32_t bad = __ballot_sync(0xffffffffu, !(b >= 0 && b < i));
    const int np = min(km1, __ffs(bad) - 1);
    if (np < 2) continue;  // the own-block kernel reads a lone partial where it is
    float M = lane < np ? lq : -INFINITY;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    const float wl = lane < np ? __expf(lq - M) : 0.f;
    float L = wl;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    float acc[kDL];
#pragma unroll
    for (int x = 0; x < kDL; ++x) acc[x] = 0.f;
#pragma unroll
    for (int q = 0; q < kMaxTopK - 1; ++q) {
      const float w = __shfl_sync(0xffffffffu, wl, q);
      if (q < np) {
#pragma unroll
        for (int x = 0; x < kDL / 2; ++x) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&raw[q][x]));
          acc[2 * x] = fmaf(w, f.x, acc[2 * x]);
          acc[2 * x + 1] = fmaf(w, f.y, acc[2 * x + 1]);
        }
      }
    }
    const float inv = 1.f / L;
    __half2* dst = reinterpret_cast<__half2*>(mo + row * D + lane * kDL);
#pragma unroll
    for (int x = 0; x < kDL / 2; ++x) dst[x] = __floats2half2_rn(acc[2 * x] * inv, acc[2 * x + 1] * inv);
    if (lane == 0) mlse[row] = M + __logf(L);
  }
}
}  // namespace

cudaError_t launch_attn_self(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                             const __nv_bfloat16* V, const int32_t* sel, const Work& w,
                             __nv_bfloat16* O, float* LSE, cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  int premerged = 0;
  if (premerge_used(g)) {
    const int64_t rows = (int64_t)g.T * g.Hq;
    const int64_t want = (rows + 7) / 8;
    const unsigned blocks = (unsigned)(want < 148 * 64 ? want : 148 * 64);
    if (g.D == 64) premerge_kernel<64><<<blocks, 256, 0, st>>>(g, sel, w.part_o, w.part_lse, w.merged_o, w.merged_lse);
    else premerge_kernel<128><<<blocks, 256, 0, st>>>(g, sel, w.part_o, w.part_lse, w.merged_o, w.merged_lse);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    premerged = 1;
  }
  return launch_own_tiles(g, Q, K, V, sel, w, O, LSE, premerged, st);
}

cudaError_t launch_attn_naive(const Geom& g, const __nv_bfloat16* Q, const __nv_bfloat16* K,
                              const __nv_bfloat16* V, const int32_t* sel, __nv_bfloat16* O, float* LSE,
                              cudaStream_t st) {
  if (g.T == 0) return cudaSuccess;
  return launch_naive_tiles(g, Q, K, V, sel, O, LSE, st);
}

int launches_per_forward(const Geom& g) {
  // pool + gate (Kbar split, scores/top-k) + (route count, scan, scatter + past attention
  // when top_k > 1) + (partial pre-merge when a row can have more than two partials) +
  // own block/merge
  return 3 + (g.k > 1 ? 4 : 0) + (premerge_used(g) ? 1 : 0) + 1;
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
