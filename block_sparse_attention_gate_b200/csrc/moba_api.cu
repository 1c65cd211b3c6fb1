// C ABI of the MoBA causal-prefill library: argument validation, workspace carve-up and
// the launch sequence (pool -> gate -> route -> block attention + merge).  Nothing here
// allocates or synchronises; every kernel is enqueued on the caller's stream.
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <mutex>

#include "moba.h"
#include "moba_internal.cuh"
#include "sm100.cuh"

// Device error word: kernels OR a code into it when a bounded wait gives up.
__device__ int g_moba_device_error = 0;

// One thread waits on an mbarrier phase that nothing completes, through the same bounded wait
// the tensor-core kernels use: the wait gives up, sets the error word and the kernel returns.
__global__ void bounded_wait_selftest_kernel(int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    moba::mbar_init(&bar, 1);
    moba::fence_mbar_init();
    moba::mbar_wait(&bar, 0, err);
  }
}

namespace {

thread_local char g_err[512] = "";

void set_err(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
}

moba_status fail(moba_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

moba_status cuda_fail(cudaError_t e, const char* where) {
  set_err("%s: %s", where, cudaGetErrorString(e));
  return MOBA_ERR_CUDA;
}

constexpr int64_t kI32Max = 2147483647LL;

// Validate the parameters and derive the kernels' geometry (host only).
moba_status make_geom(const moba_params* p, moba::Geom* g) {
  if (!p) return fail(MOBA_ERR_INVALID_ARG, "params is NULL");
  if (p->num_seqs < 1) return fail(MOBA_ERR_INVALID_ARG, "num_seqs must be >= 1 (got %d)", p->num_seqs);
  if (p->num_seqs > 65535) return fail(MOBA_ERR_UNSUPPORTED, "num_seqs must be <= 65535 (got %d)", p->num_seqs);
  if (p->num_q_heads < 1 || p->num_kv_heads < 1 || p->num_q_heads % p->num_kv_heads)
    return fail(MOBA_ERR_INVALID_ARG, "num_q_heads (%d) must be a positive multiple of num_kv_heads (%d)",
                p->num_q_heads, p->num_kv_heads);
  if (p->head_dim != 64 && p->head_dim != 128)
    return fail(MOBA_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", p->head_dim);
  if (p->block_size < 128 || p->block_size % 128 || p->block_size > 8192)
    return fail(MOBA_ERR_UNSUPPORTED, "block_size must be a multiple of 128 in [128, 8192] (got %d)",
                p->block_size);
  if (p->top_k < 1 || p->top_k > moba::kMaxTopK)
    return fail(MOBA_ERR_UNSUPPORTED, "top_k must be in [1, %d] (got %d)", moba::kMaxTopK, p->top_k);
  if ((int64_t)p->num_kv_heads * p->head_dim > 16384)
    return fail(MOBA_ERR_UNSUPPORTED, "num_kv_heads * head_dim must be <= 16384");
  int64_t T = 0, maxlen = 0;
  if (p->cu_seqlens_host) {
    if (!p->cu_seqlens) return fail(MOBA_ERR_INVALID_ARG, "cu_seqlens (device) is NULL but the host copy is not");
    if (p->cu_seqlens_host[0] != 0) return fail(MOBA_ERR_INVALID_ARG, "cu_seqlens[0] must be 0");
    for (int s = 0; s < p->num_seqs; ++s) {
      int64_t len = (int64_t)p->cu_seqlens_host[s + 1] - p->cu_seqlens_host[s];
      if (len < 0) return fail(MOBA_ERR_INVALID_ARG, "cu_seqlens must be nondecreasing (at %d)", s);
      if (len > maxlen) maxlen = len;
    }
    T = p->cu_seqlens_host[p->num_seqs];
    if (((uintptr_t)p->cu_seqlens) & 3) return fail(MOBA_ERR_ALIGNMENT, "cu_seqlens (device) misaligned");
  } else {
    if (p->cu_seqlens) return fail(MOBA_ERR_INVALID_ARG, "cu_seqlens given without cu_seqlens_host");
    if (p->max_seqlen < 0) return fail(MOBA_ERR_INVALID_ARG, "max_seqlen must be >= 0");
    maxlen = p->max_seqlen;
    T = (int64_t)p->num_seqs * maxlen;
  }
  if (T > kI32Max) return fail(MOBA_ERR_UNSUPPORTED, "total tokens exceed 2^31-1");
  const int64_t MB = (maxlen + p->block_size - 1) / p->block_size;
  if (MB > 16384) return fail(MOBA_ERR_UNSUPPORTED, "more than 16384 blocks in one sequence");
  if (T * p->num_q_heads * p->top_k > kI32Max)
    return fail(MOBA_ERR_UNSUPPORTED, "T * Hq * top_k exceeds 2^31-1");
  g->cu = p->cu_seqlens_host ? p->cu_seqlens : nullptr;
  g->num_seqs = p->num_seqs;
  g->L = (int32_t)(p->cu_seqlens_host ? 0 : maxlen);
  g->T = (int32_t)T;
  g->Hq = p->num_q_heads;
  g->Hkv = p->num_kv_heads;
  g->G = p->num_q_heads / p->num_kv_heads;
  g->D = p->head_dim;
  g->bs = p->block_size;
  g->MB = (int32_t)MB;
  g->k = p->top_k;
  g->scale = p->softmax_scale > 0.f ? p->softmax_scale : 1.0f / sqrtf((float)p->head_dim);
  g->scale_log2 = g->scale * 1.4426950408889634f;
  g->nbk = (int64_t)p->num_kv_heads * p->num_seqs * MB;
  g->R = T * p->num_q_heads * (p->top_k - 1);
  return MOBA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace carve-up; with base == nullptr only the size is computed.
size_t carve(const moba::Geom& g, char* base, moba::Work* w) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* ptr = base ? base + off : nullptr;
    off += align256(bytes);
    return ptr;
  };
  moba::Work x;
  x.counts = (int32_t*)take(sizeof(int32_t) * (size_t)g.nbk);
  x.cursors = (int32_t*)take(sizeof(int32_t) * (size_t)g.nbk);
  x.tile_off = (int32_t*)take(sizeof(int32_t) * (size_t)(g.nbk + 1));
  x.tile_bucket = (int32_t*)take(sizeof(int32_t) * (size_t)moba::past_tiles(g));
  x.rows = (int32_t*)take(sizeof(int32_t) * (size_t)moba::past_tiles(g) * moba::kPastTileRows);
  x.part_o = (__half*)take(sizeof(__half) * (size_t)g.R * g.D);
  x.part_lse = (float*)take(sizeof(float) * (size_t)g.R);
  const size_t nmerged = moba::premerge_used(g) ? (size_t)g.T * g.Hq : 0;
  x.merged_o = (__half*)take(sizeof(__half) * nmerged * g.D);
  x.merged_lse = (float*)take(sizeof(float) * nmerged);
  x.kbar = (float*)take(sizeof(float) * (size_t)g.num_seqs * g.MB * g.Hkv * g.D);
  x.sel = (int32_t*)take(sizeof(int32_t) * (size_t)g.T * g.Hq * g.k);
  x.kbar_hi = (__nv_bfloat16*)take(2 * (size_t)g.num_seqs * g.MB * g.Hkv * g.D);
  x.kbar_lo = (__nv_bfloat16*)take(2 * (size_t)g.num_seqs * g.MB * g.Hkv * g.D);
  x.kbar_n2 = (float*)take(sizeof(float) * (size_t)g.num_seqs * g.MB * g.Hkv);
  x.bytes = off;
  if (w) *w = x;
  return off;
}

constexpr int kMaxDevices = 64;

// Device address of a __device__ variable, looked up once per device (with that device
// current) by the first caller; concurrent first callers on other host threads wait for it.
// The host-side name of a __device__ variable is only a stand-in, never a device address.
// The cached address belongs to the device's primary context: it is not valid after
// cudaDeviceReset on that device.
struct SymbolAddress {
  std::once_flag once[kMaxDevices];
  void* ptr[kMaxDevices] = {};
  cudaError_t err[kMaxDevices] = {};
};

template <typename Sym>
cudaError_t symbol_address(SymbolAddress& cache, int dev, const Sym& symbol, void** out) {
  std::call_once(cache.once[dev], [&] { cache.err[dev] = cudaGetSymbolAddress(&cache.ptr[dev], symbol); });
  *out = cache.ptr[dev];
  return cache.err[dev];
}

SymbolAddress g_err_addr;  // g_moba_device_error

// Checks that the current device is an sm_100 part and binds the device error word's
// address (looked up once per device with that device current) into the geometry.
moba_status check_device(moba::Geom* g) {
  int dev = 0, major = 0, minor = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
  if (major != 10 || minor != 0)
    return fail(MOBA_ERR_DEVICE, "device %d is sm_%d%d; this library is built for sm_100a", dev, major, minor);
  if (dev < 0 || dev >= kMaxDevices) return fail(MOBA_ERR_DEVICE, "device ordinal %d out of range", dev);
  void* p = nullptr;
  e = symbol_address(g_err_addr, dev, g_moba_device_error, &p);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(device error word)");
  g->err = static_cast<int*>(p);
  return MOBA_OK;
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15) == 0; }

moba_status check_ptr(const void* ptr, const char* name, bool needed) {
  if (!needed) return MOBA_OK;
  if (!ptr) return fail(MOBA_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(ptr)) return fail(MOBA_ERR_ALIGNMENT, "%s is not 16-byte aligned", name);
  return MOBA_OK;
}

moba_status check_ws(const moba::Geom& g, void* ws, size_t bytes, moba::Work* w) {
  const size_t need = carve(g, nullptr, nullptr);
  if (need && !ws) return fail(MOBA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (((uintptr_t)ws) & 255) return fail(MOBA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (bytes < need) return fail(MOBA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", bytes, need);
  carve(g, (char*)ws, w);
  return MOBA_OK;
}

#define MOBA_TRY(x)                      \
  do {                                   \
    moba_status _s = (x);                \
    if (_s != MOBA_OK) return _s;        \
  } while (0)

}  // namespace

extern "C" {

size_t moba_kbar_elems(const moba_params* p) {
  moba::Geom g;
  if (make_geom(p, &g) != MOBA_OK) return 0;
  return (size_t)g.num_seqs * g.MB * g.Hkv * g.D;
}

size_t moba_workspace_size(const moba_params* p) {
  moba::Geom g;
  if (make_geom(p, &g) != MOBA_OK) return 0;
  return carve(g, nullptr, nullptr);
}

moba_status moba_pool_keys(const moba_params* p, const void* K, float* Kbar, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0 || g.MB == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(Kbar, "Kbar", true));
  MOBA_TRY(check_device(&g));
  cudaError_t e = moba::launch_pool(g, (const __nv_bfloat16*)K, Kbar, (cudaStream_t)stream);
  return e == cudaSuccess ? MOBA_OK : cuda_fail(e, "pool launch");
}

moba_status moba_gate_topk(const moba_params* p, const void* Q, const float* Kbar, int32_t* sel,
                           void* workspace, size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(Kbar, "Kbar", true));
  MOBA_TRY(check_ptr(sel, "sel", true));
  moba::Work w;
  MOBA_TRY(check_ws(g, workspace, workspace_bytes, &w));
  MOBA_TRY(check_device(&g));
  cudaError_t e = moba::launch_gate(g, (const __nv_bfloat16*)Q, Kbar, sel, w, (cudaStream_t)stream);
  return e == cudaSuccess ? MOBA_OK : cuda_fail(e, "gate launch");
}

static moba_status attn_stages(const moba::Geom& g, const void* Q, const void* K, const void* V,
                               const int32_t* sel, const moba::Work& w, void* O, float* LSE,
                               cudaStream_t st, int which /* 1 route, 2 past, 4 self */) {
  cudaError_t e = cudaSuccess;
  if ((which & 1) && g.k > 1) {
    e = moba::launch_route(g, sel, w, st);
    if (e != cudaSuccess) return cuda_fail(e, "route launch");
  }
  if (which & 2) {
    e = moba::launch_attn_past(g, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, w, st);
    if (e != cudaSuccess) return cuda_fail(e, "past-block attention launch");
  }
  if (which & 4) {
    e = moba::launch_attn_self(g, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V, sel,
                               w, (__nv_bfloat16*)O, LSE, st);
    if (e != cudaSuccess) return cuda_fail(e, "own-block attention launch");
  }
  return MOBA_OK;
}

moba_status moba_attn_fwd(const moba_params* p, const void* Q, const void* K, const void* V,
                          const int32_t* sel, void* workspace, size_t workspace_bytes, void* O,
                          float* LSE, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(V, "V", true));
  MOBA_TRY(check_ptr(sel, "sel", true));
  MOBA_TRY(check_ptr(O, "O", true));
  MOBA_TRY(check_ptr(LSE, "LSE", true));
  moba::Work w;
  MOBA_TRY(check_ws(g, workspace, workspace_bytes, &w));
  MOBA_TRY(check_device(&g));
  return attn_stages(g, Q, K, V, sel, w, O, LSE, (cudaStream_t)stream, 7);
}

moba_status moba_route(const moba_params* p, const int32_t* sel, void* workspace, size_t workspace_bytes,
                       void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(sel, "sel", true));
  moba::Work w;
  MOBA_TRY(check_ws(g, workspace, workspace_bytes, &w));
  MOBA_TRY(check_device(&g));
  return attn_stages(g, nullptr, nullptr, nullptr, sel, w, nullptr, nullptr, (cudaStream_t)stream, 1);
}

moba_status moba_attn_past(const moba_params* p, const void* Q, const void* K, const void* V, void* workspace,
                           size_t workspace_bytes, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(V, "V", true));
  moba::Work w;
  MOBA_TRY(check_ws(g, workspace, workspace_bytes, &w));
  MOBA_TRY(check_device(&g));
  return attn_stages(g, Q, K, V, nullptr, w, nullptr, nullptr, (cudaStream_t)stream, 2);
}

moba_status moba_attn_self_merge(const moba_params* p, const void* Q, const void* K, const void* V,
                                 const int32_t* sel, void* workspace, size_t workspace_bytes, void* O,
                                 float* LSE, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(V, "V", true));
  MOBA_TRY(check_ptr(sel, "sel", true));
  MOBA_TRY(check_ptr(O, "O", true));
  MOBA_TRY(check_ptr(LSE, "LSE", true));
  moba::Work w;
  MOBA_TRY(check_ws(g, workspace, workspace_bytes, &w));
  MOBA_TRY(check_device(&g));
  return attn_stages(g, Q, K, V, sel, w, O, LSE, (cudaStream_t)stream, 4);
}

moba_status moba_attn_naive(const moba_params* p, const void* Q, const void* K, const void* V,
                            const int32_t* sel, void* O, float* LSE, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(V, "V", true));
  MOBA_TRY(check_ptr(sel, "sel", true));
  MOBA_TRY(check_ptr(O, "O", true));
  MOBA_TRY(check_ptr(LSE, "LSE", true));
  MOBA_TRY(check_device(&g));
  cudaError_t e = moba::launch_attn_naive(g, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K,
                                          (const __nv_bfloat16*)V, sel, (__nv_bfloat16*)O, LSE,
                                          (cudaStream_t)stream);
  return e == cudaSuccess ? MOBA_OK : cuda_fail(e, "mask-based attention launch");
}

}  // extern "C"

namespace {
// Decode needs every sequence to hold at least the new token.
moba_status check_decode_lengths(const moba_params* p) {
  if (p->cu_seqlens_host) {
    for (int s = 0; s < p->num_seqs; ++s)
      if (p->cu_seqlens_host[s + 1] - p->cu_seqlens_host[s] < 1)
        return fail(MOBA_ERR_INVALID_ARG, "decode: sequence %d is empty (the cache must hold the new token)", s);
  } else if (p->max_seqlen < 1) {
    return fail(MOBA_ERR_INVALID_ARG, "decode: max_seqlen must be >= 1");
  }
  return MOBA_OK;
}

struct DecodeWork {
  float* part_o;
  float* part_lse;
  int32_t* sel;
  size_t bytes;
};

DecodeWork carve_decode(const moba::Geom& g, char* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* ptr = base ? base + off : nullptr;
    off += align256(bytes);
    return ptr;
  };
  const size_t units = (size_t)g.num_seqs * g.Hq * g.k;
  DecodeWork w;
  w.part_o = (float*)take(units * g.D * sizeof(float));
  w.part_lse = (float*)take(units * sizeof(float));
  w.sel = (int32_t*)take(units * sizeof(int32_t));
  w.bytes = off;
  return w;
}
}  // namespace

extern "C" {

}  // extern "C"

namespace {
// Backward workspace: the routing arrays (as the forward's), Dp, fp32 dQ partials.
struct BwdWork {
  moba::Work route;
  float* Dp;
  float* dq_part;
  size_t bytes;
};

BwdWork carve_bwd(const moba::Geom& g, char* base) {
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* ptr = base ? base + off : nullptr;
    off += align256(bytes);
    return ptr;
  };
  BwdWork w;
  moba::Work x{};
  x.counts = (int32_t*)take(sizeof(int32_t) * (size_t)g.nbk);
  x.cursors = (int32_t*)take(sizeof(int32_t) * (size_t)g.nbk);
  x.tile_off = (int32_t*)take(sizeof(int32_t) * (size_t)(g.nbk + 1));
  x.tile_bucket = (int32_t*)take(sizeof(int32_t) * (size_t)moba::past_tiles(g));
  x.rows = (int32_t*)take(sizeof(int32_t) * (size_t)moba::past_tiles(g) * moba::kPastTileRows);
  w.route = x;
  w.Dp = (float*)take(sizeof(float) * (size_t)g.T * g.Hq);
  w.dq_part = (float*)take(sizeof(float) * (size_t)g.R * g.D);
  w.bytes = off;
  return w;
}
}  // namespace

extern "C" {

size_t moba_bwd_workspace_size(const moba_params* p) {
  moba::Geom g;
  if (make_geom(p, &g) != MOBA_OK) return 0;
  return carve_bwd(g, nullptr).bytes;
}

moba_status moba_attn_bwd(const moba_params* p, const void* Q, const void* K, const void* V, const void* O,
                          const float* LSE, const void* dO, const int32_t* sel, void* workspace,
                          size_t workspace_bytes, void* dQ, void* dK, void* dV, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(V, "V", true));
  MOBA_TRY(check_ptr(O, "O", true));
  MOBA_TRY(check_ptr(LSE, "LSE", true));
  MOBA_TRY(check_ptr(dO, "dO", true));
  MOBA_TRY(check_ptr(sel, "sel", true));
  MOBA_TRY(check_ptr(dQ, "dQ", true));
  MOBA_TRY(check_ptr(dK, "dK", true));
  MOBA_TRY(check_ptr(dV, "dV", true));
  const size_t need = carve_bwd(g, nullptr).bytes;
  if (!workspace) return fail(MOBA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (((uintptr_t)workspace) & 255) return fail(MOBA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (workspace_bytes < need) return fail(MOBA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
  MOBA_TRY(check_device(&g));
  BwdWork w = carve_bwd(g, (char*)workspace);
  cudaError_t e = moba::launch_attn_bwd(g, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
                                        (const __nv_bfloat16*)O, LSE, (const __nv_bfloat16*)dO, sel, w.route, w.Dp,
                                        w.dq_part, (__nv_bfloat16*)dQ, (__nv_bfloat16*)dK, (__nv_bfloat16*)dV,
                                        (cudaStream_t)stream);
  return e == cudaSuccess ? MOBA_OK : cuda_fail(e, "backward launch");
}

moba_status moba_pool_last_block(const moba_params* p, const void* K, float* Kbar, void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0 || g.MB == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(Kbar, "Kbar", true));
  MOBA_TRY(check_device(&g));
  cudaError_t e = moba::launch_pool_last(g, (const __nv_bfloat16*)K, Kbar, (cudaStream_t)stream);
  return e == cudaSuccess ? MOBA_OK : cuda_fail(e, "pool (last block) launch");
}

size_t moba_decode_workspace_size(const moba_params* p) {
  moba::Geom g;
  if (make_geom(p, &g) != MOBA_OK) return 0;
  return carve_decode(g, nullptr).bytes;
}

moba_status moba_decode_fwd(const moba_params* p, const void* Q, const void* K, const void* V, const float* Kbar,
                            int32_t* sel, void* workspace, size_t workspace_bytes, void* O, float* LSE,
                            void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  MOBA_TRY(check_decode_lengths(p));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(V, "V", true));
  MOBA_TRY(check_ptr(Kbar, "Kbar", true));
  MOBA_TRY(check_ptr(sel, "sel", sel != nullptr));
  MOBA_TRY(check_ptr(O, "O", true));
  MOBA_TRY(check_ptr(LSE, "LSE", true));
  const size_t need = carve_decode(g, nullptr).bytes;
  if (!workspace) return fail(MOBA_ERR_WORKSPACE, "workspace is NULL (%zu bytes needed)", need);
  if (((uintptr_t)workspace) & 255) return fail(MOBA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (workspace_bytes < need) return fail(MOBA_ERR_WORKSPACE, "workspace has %zu bytes, %zu needed", workspace_bytes, need);
  MOBA_TRY(check_device(&g));
  DecodeWork w = carve_decode(g, (char*)workspace);
  cudaError_t e = moba::launch_decode(g, (const __nv_bfloat16*)Q, (const __nv_bfloat16*)K, (const __nv_bfloat16*)V,
                                      Kbar, sel ? sel : w.sel, w.part_o, w.part_lse, (__nv_bfloat16*)O, LSE,
                                      (cudaStream_t)stream);
  return e == cudaSuccess ? MOBA_OK : cuda_fail(e, "decode launch");
}

int moba_launches_per_forward(const moba_params* p) {
  moba::Geom g;
  if (make_geom(p, &g) != MOBA_OK) return -1;
  if (g.T == 0) return 0;
  return moba::launches_per_forward(g);
}

moba_status moba_fwd(const moba_params* p, const void* Q, const void* K, const void* V, float* Kbar,
                     int32_t* sel, void* workspace, size_t workspace_bytes, void* O, float* LSE,
                     void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(K, "K", true));
  MOBA_TRY(check_ptr(V, "V", true));
  MOBA_TRY(check_ptr(O, "O", true));
  MOBA_TRY(check_ptr(LSE, "LSE", true));
  MOBA_TRY(check_ptr(Kbar, "Kbar", Kbar != nullptr));
  MOBA_TRY(check_ptr(sel, "sel", sel != nullptr));
  moba::Work w;
  MOBA_TRY(check_ws(g, workspace, workspace_bytes, &w));
  MOBA_TRY(check_device(&g));
  float* kb = Kbar ? Kbar : w.kbar;
  int32_t* sl = sel ? sel : w.sel;
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e = moba::launch_pool(g, (const __nv_bfloat16*)K, kb, st);
  if (e != cudaSuccess) return cuda_fail(e, "pool launch");
  e = moba::launch_gate(g, (const __nv_bfloat16*)Q, kb, sl, w, st);
  if (e != cudaSuccess) return cuda_fail(e, "gate launch");
  return attn_stages(g, Q, K, V, sl, w, O, LSE, st, 7);
}

// ------------------------------------------------------------------ host-buffer forward
namespace {

// Parameters of one KV-head group as a problem of its own (G query heads, one KV head).
moba_params group_params(const moba_params* p) {
  moba_params q = *p;
  q.num_q_heads = p->num_q_heads / p->num_kv_heads;
  q.num_kv_heads = 1;
  return q;
}

struct HostSlot {
  char* Q;
  char* K;
  char* V;
  char* O;
  float* LSE;
  char* ws;
  size_t ws_bytes;
  size_t bytes;
};

// Device staging of one slot: Q, K, V, O, LSE of one group plus that group's workspace.
HostSlot carve_slot(const moba::Geom& gg, size_t ws_bytes, char* base) {
  HostSlot h;
  size_t off = 0;
  auto take = [&](size_t bytes) -> char* {
    char* ptr = base ? base + off : nullptr;
    off += align256(bytes);
    return ptr;
  };
  const size_t T = (size_t)gg.T, D = (size_t)gg.D, G = (size_t)gg.Hq;
  h.Q = take(T * G * D * 2);
  h.K = take(T * D * 2);
  h.V = take(T * D * 2);
  h.O = take(T * G * D * 2);
  h.LSE = (float*)take(T * G * 4);
  h.ws = take(ws_bytes);
  h.ws_bytes = ws_bytes;
  h.bytes = off;
  return h;
}

}  // namespace

size_t moba_host_staging_size(const moba_params* p, int nslots) {
  moba::Geom g;
  if (make_geom(p, &g) != MOBA_OK || nslots < 1) return 0;
  moba_params q = group_params(p);
  moba::Geom gg;
  if (make_geom(&q, &gg) != MOBA_OK) return 0;
  const size_t ws = carve(gg, nullptr, nullptr);
  return (size_t)nslots * carve_slot(gg, ws, nullptr).bytes;
}

moba_status moba_fwd_host(const moba_params* p, const void* Q, const void* K, const void* V, void* O, float* LSE,
                          void* staging, size_t staging_bytes, void* const* streams, int nstreams) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  if (!Q || !K || !V || !O || !LSE) return fail(MOBA_ERR_INVALID_ARG, "a host buffer is NULL");
  if (!streams || nstreams < 1) return fail(MOBA_ERR_INVALID_ARG, "need at least one stream");
  const size_t need = moba_host_staging_size(p, nstreams);
  if (!staging || (((uintptr_t)staging) & 255)) return fail(MOBA_ERR_WORKSPACE, "staging missing or not 256-byte aligned");
  if (staging_bytes < need) return fail(MOBA_ERR_WORKSPACE, "staging has %zu bytes, %zu needed", staging_bytes, need);
  moba_params q = group_params(p);
  moba::Geom gg;
  MOBA_TRY(make_geom(&q, &gg));
  MOBA_TRY(check_device(&gg));
  const size_t ws = carve(gg, nullptr, nullptr);
  const size_t slot_bytes = carve_slot(gg, ws, nullptr).bytes;
  const size_t T = (size_t)g.T, D = (size_t)g.D, G = (size_t)gg.Hq;
  const size_t Hq = (size_t)g.Hq, Hkv = (size_t)g.Hkv;
  for (int grp = 0; grp < g.Hkv; ++grp) {
    const int slot = grp % nstreams;
    cudaStream_t st = (cudaStream_t)streams[slot];
    HostSlot h = carve_slot(gg, ws, (char*)staging + (size_t)slot * slot_bytes);
    const char* qh = (const char*)Q + (size_t)grp * G * D * 2;
    const char* kh = (const char*)K + (size_t)grp * D * 2;
    const char* vh = (const char*)V + (size_t)grp * D * 2;
    cudaError_t e = cudaMemcpy2DAsync(h.Q, G * D * 2, qh, Hq * D * 2, G * D * 2, T, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(h.K, D * 2, kh, Hkv * D * 2, D * 2, T, cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(h.V, D * 2, vh, Hkv * D * 2, D * 2, T, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy");
    moba::Work w;
    carve(gg, h.ws, &w);
    e = moba::launch_pool(gg, (const __nv_bfloat16*)h.K, w.kbar, st);
    if (e != cudaSuccess) return cuda_fail(e, "pool launch");
    e = moba::launch_gate(gg, (const __nv_bfloat16*)h.Q, w.kbar, w.sel, w, st);
    if (e != cudaSuccess) return cuda_fail(e, "gate launch");
    MOBA_TRY(attn_stages(gg, h.Q, h.K, h.V, w.sel, w, h.O, h.LSE, st, 7));
    char* oh = (char*)O + (size_t)grp * G * D * 2;
    float* lh = LSE + (size_t)grp * G;
    e = cudaMemcpy2DAsync(oh, Hq * D * 2, h.O, G * D * 2, G * D * 2, T, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaMemcpy2DAsync(lh, Hq * 4, h.LSE, G * 4, G * 4, T, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy");
  }
  return MOBA_OK;
}

const char* moba_status_string(int status) {
  switch (status) {
    case MOBA_OK: return "ok";
    case MOBA_ERR_INVALID_ARG: return "invalid argument";
    case MOBA_ERR_UNSUPPORTED: return "unsupported size";
    case MOBA_ERR_ALIGNMENT: return "misaligned pointer";
    case MOBA_ERR_WORKSPACE: return "workspace missing or too small";
    case MOBA_ERR_CUDA: return "CUDA error";
    case MOBA_ERR_DEVICE: return "unsupported device";
    default: return "unknown status";
  }
}

const char* moba_last_error(void) { return g_err; }

moba_status moba_selftest_bounded_wait(int32_t* device_error) {
  g_err[0] = 0;
  if (!device_error) return fail(MOBA_ERR_INVALID_ARG, "device_error is NULL");
  moba::Geom g;
  MOBA_TRY(check_device(&g));
  cudaError_t e = cudaMemset(g.err, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  bounded_wait_selftest_kernel<<<1, 32>>>(g.err);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "self-test");
  int v = 0;
  e = cudaMemcpy(&v, g.err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  e = cudaMemset(g.err, 0, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  *device_error = v;
  return MOBA_OK;
}

moba_status moba_read_device_error(int32_t* value, int clear) {
  g_err[0] = 0;
  if (!value) return fail(MOBA_ERR_INVALID_ARG, "value is NULL");
  moba::Geom g;
  MOBA_TRY(check_device(&g));
  int v = 0;
  cudaError_t e = cudaMemcpy(&v, g.err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (clear) {
    e = cudaMemset(g.err, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  }
  *value = v;
  return MOBA_OK;
}

// ---------------------------------------------------------------------------------------
// Gate without caller scratch.  The tensor-core gate needs scratch for the bf16 hi/lo split of
// the pooled keys; this variant keeps it in a fixed device array compiled into the library,
// so the caller passes only inputs and outputs and nothing here allocates.
}  // extern "C"

namespace {
constexpr size_t kNoAllocMaxKbarElems = (size_t)1 << 21;  // hi + lo: 2 x 2^21 bf16 = 8 MiB
// Squared norms, one fp32 per pooled-key row (head_dim >= 64: at most 2^15 rows), stored
// after hi and lo as pairs of bf16 slots.
constexpr size_t kNoAllocNormSlots = 2 * (kNoAllocMaxKbarElems / 64);
}  // namespace

static __device__ __align__(256) __nv_bfloat16 g_gate_scratch[2 * kNoAllocMaxKbarElems + kNoAllocNormSlots];

namespace {
SymbolAddress g_gate_scratch_addr;

// Device address of g_gate_scratch on the current device, looked up once per device (the
// host-side name of the array is only a stand-in, never a device address).
moba_status gate_scratch(__nv_bfloat16** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(MOBA_ERR_DEVICE, "device ordinal %d out of range", dev);
  void* ptr = nullptr;
  e = symbol_address(g_gate_scratch_addr, dev, g_gate_scratch, &ptr);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(gate scratch)");
  *out = static_cast<__nv_bfloat16*>(ptr);
  return MOBA_OK;
}
}  // namespace

extern "C" {

moba_status moba_gate_topk_noalloc(const moba_params* p, const void* Q, const float* Kbar, int32_t* sel,
                                   void* stream) {
  g_err[0] = 0;
  moba::Geom g;
  MOBA_TRY(make_geom(p, &g));
  if (g.T == 0) return MOBA_OK;
  const size_t elems = (size_t)g.num_seqs * g.MB * g.Hkv * g.D;
  if (elems > kNoAllocMaxKbarElems)
    return fail(MOBA_ERR_UNSUPPORTED,
                "moba_gate_topk_noalloc: num_seqs * ceil(max_seqlen / block_size) * num_kv_heads * head_dim = "
                "%zu exceeds the built-in scratch limit of %zu; use moba_gate_topk with a workspace",
                elems, kNoAllocMaxKbarElems);
  MOBA_TRY(check_ptr(Q, "Q", true));
  MOBA_TRY(check_ptr(Kbar, "Kbar", true));
  MOBA_TRY(check_ptr(sel, "sel", true));
  MOBA_TRY(check_device(&g));
  __nv_bfloat16* scratch = nullptr;
  MOBA_TRY(gate_scratch(&scratch));
  moba::Work w{};
  w.kbar_hi = scratch;
  w.kbar_lo = scratch + kNoAllocMaxKbarElems;
  w.kbar_n2 = reinterpret_cast<float*>(scratch + 2 * kNoAllocMaxKbarElems);
  cudaError_t e = moba::launch_gate(g, (const __nv_bfloat16*)Q, Kbar, sel, w, (cudaStream_t)stream);
  return e == cudaSuccess ? MOBA_OK : cuda_fail(e, "gate launch");
}

}  // extern "C"
