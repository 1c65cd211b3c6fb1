// Definitions shared by the tensor-core attention kernels (attn_own.cu: own block + merge and
// the mask-based form; attn_past.cu: past blocks): warp roles and the register split, the
// tile and TMEM geometry, the FMA-pipe exp2, the kernels' argument block and the warp-wide
// MMA issue with 32-bit descriptor words.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include "moba_internal.cuh"
#include "sm100.cuh"

namespace moba {

namespace {

// Past-block kernel: warps 0-3 softmax tile 0, 4-7 softmax tile 1, 8 TMA, 9 MMA, 10-11 idle.
constexpr int kThreads = 384;
// Register split (setmaxnreg): the kernel is compiled for kLaunchRegs per thread; the third
// warpgroup gives registers back so the two softmax warpgroups can hold a full S row.
// 2 * 128 * kSoftmaxRegs + 128 * kOtherRegs must not exceed 384 * kLaunchRegs (checked on
// the host against the compiled register count before every launch).
constexpr uint32_t kLaunchRegs = 168;
constexpr uint32_t kSoftmaxRegs = 216;
constexpr uint32_t kOtherRegs = 72;
static_assert(2 * 128 * kSoftmaxRegs + 128 * kOtherRegs <= 384 * kLaunchRegs, "register split too large");
constexpr int kRows = 128;     // query rows per tile (M)
constexpr int kBN = 128;       // keys per chunk (N of S, K of PV)
constexpr uint32_t kTmemCols = 512;  // past-block kernel: S and O of two tiles
constexpr uint32_t kColS = 0;      // S of tile t at kColS + 128 t
constexpr uint32_t kColP = 0;      // P of tile t (bf16 pairs) aliased at S + 0 .. S + 63
constexpr uint32_t kColO = 256;    // O of tile t at kColO + 128 t
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;  // rescale O only when a row max grows by more than 2^8

// 2^x for a pair on the FMA pipe, for a share of the exponentials that would otherwise all
// queue on the MUFU unit: x = j + f with j = rint(x) (the 1.5 * 2^23 rounding trick) and
// f in [-0.5, 0.5]; 2^f from a degree-3 polynomial (relative error 7.5e-5; coefficients from
// our own iteratively reweighted least-squares fit of 2^f on that interval), 2^j added into
// the exponent field.  x is clamped to >= -126 so the exponent never wraps; below 2^-24 the
// result only has to be negligible next to the row sum, as it is.
constexpr int kPolyNum = 1, kPolyDen = 4;  // pairs (pair index mod kPolyDen) < kPolyNum use it
__device__ __forceinline__ void exp2_poly2(float& p0, float& p1, float x0, float x1) {
  constexpr float kRound = 12582912.f;  // 1.5 * 2^23
  x0 = fmaxf(x0, -126.f);
  x1 = fmaxf(x1, -126.f);
  float t0, t1, r0, r1, f0, f1, q0, q1;
  add2(t0, t1, x0, x1, kRound, kRound);
  add2(r0, r1, t0, t1, -kRound, -kRound);
  fma2(f0, f1, r0, r1, -1.f, -1.f, x0, x1);
  fma2(q0, q1, f0, f1, 0.05517132207751274f, 0.05517132207751274f, 0.24261054396629333f, 0.24261054396629333f);
  fma2(q0, q1, q0, q1, f0, f1, 0.6932609677314758f, 0.6932609677314758f);
  fma2(q0, q1, q0, q1, f0, f1, 0.9999281167984009f, 0.9999281167984009f);
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

struct AttnArgs {
  Geom g;
  const __nv_bfloat16* Q;
  const int32_t* sel;
  const int32_t* tile_off;
  const int32_t* tile_bucket;
  const int32_t* rows;
  __half* part_o;
  float* part_lse;
  __nv_bfloat16* O;
  float* LSE;
  int premerged;       // own mode: rows with two or more past partials have them folded in mo/mlse
  const __half* mo;    // [T * Hq, D] folded partial of each such row
  const float* mlse;   // [T * Hq] its LSE
};


}  // namespace

}  // namespace moba
