/*
 * moba.h -- C ABI of the MoBA (Mixture of Block Attention) causal-prefill library
 * for NVIDIA B200 (sm_100a).
 *
 * MoBA splits the keys of every sequence into equal blocks, mean-pools each
 * block's keys, lets every query score the pooled keys of its past blocks with a
 * parameter-free dot product, keeps its own block plus the best-scoring past
 * blocks (top_k in all), runs exact softmax attention over the chosen blocks only
 * (causal inside its own block) and merges the per-block results by online
 * softmax.  Sources: the MoBA project README ("MoBA: Mixture of Block Attention for
 * Long-Context LLMs", gittoolsai.com mirror: "Trainable Block Sparse Attention",
 * "Parameter-less Gating Mechanism", FAQ of GitHub issue #27), and the youleyou.com
 * article "Kimi发布MoBA突破性实现无限上下文" (sections "MoBA：基于块的混合注意力机制"
 * and "PyTorch实现关键要点").
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller, 16-byte aligned,
 *    contiguous, row-major.  Q is [T, Hq, D] bf16; K and V are [T, Hkv, D] bf16;
 *    T = total tokens of the packed batch (varlen packing by cu_seqlens).
 *  - The library never allocates, never synchronises the host, and enqueues its
 *    kernels asynchronously on `stream` (a cudaStream_t passed as void*; NULL is the
 *    legacy default stream).  Scratch comes from the caller's `workspace`.
 *  - Argument errors are reported before anything is enqueued.  A failed launch
 *    returns MOBA_ERR_CUDA; moba_last_error() then holds a message (per thread).
 *  - Block b of sequence s covers tokens [cu[s] + b*bs, min(cu[s] + (b+1)*bs, cu[s+1])).
 *    Block indices in `sel` are local to the sequence.
 *  - Kbar is laid out [num_seqs, MB, Hkv, D] fp32 with MB = ceil(max_seqlen / bs)
 *    (blocks past a sequence's end are written as zeros).
 *  - LSE is the natural-log log-sum-exp of the scaled logits, fp32 [T, Hq].
 */
#ifndef MOBA_H_
#define MOBA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOBA_API __attribute__((visibility("default")))
#else
#define MOBA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOBA_OK = 0,
  MOBA_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent cu_seqlens */
  MOBA_ERR_UNSUPPORTED = 2, /* a size the kernels do not handle (head_dim, block_size, top_k) */
  MOBA_ERR_ALIGNMENT = 3,   /* a device pointer is not 16-byte aligned */
  MOBA_ERR_WORKSPACE = 4,   /* workspace missing, too small or not 256-byte aligned */
  MOBA_ERR_CUDA = 5,        /* a CUDA runtime call or a kernel launch failed */
  MOBA_ERR_DEVICE = 6       /* the current device is not an sm_100 (B200-class) GPU */
} moba_status;

typedef struct {
  int32_t num_seqs;               /* >= 1 */
  const int32_t* cu_seqlens_host; /* HOST, num_seqs+1 offsets, [0] = 0, nondecreasing;
                                     NULL: num_seqs sequences of max_seqlen tokens each */
  const int32_t* cu_seqlens;      /* DEVICE copy of the same offsets (NULL iff the host copy is) */
  int32_t max_seqlen;             /* used only when cu_seqlens_host is NULL */
  int32_t num_q_heads;            /* Hq, a multiple of num_kv_heads (GQA group G = Hq/Hkv) */
  int32_t num_kv_heads;           /* Hkv */
  int32_t head_dim;               /* D: 64 or 128 */
  int32_t block_size;             /* bs: a multiple of 128, at most 8192 */
  int32_t top_k;                  /* blocks per query including its own block: 1..16 */
  float softmax_scale;            /* <= 0 means 1/sqrt(head_dim) */
} moba_params;

/* Number of fp32 elements of Kbar: num_seqs * MB * Hkv * D (0 if params are invalid). */
MOBA_API size_t moba_kbar_elems(const moba_params* p);

/* Bytes of workspace that moba_gate_topk, moba_attn_fwd and moba_fwd need (host only,
 * no CUDA call).  Returns 0 if params are invalid. */
MOBA_API size_t moba_workspace_size(const moba_params* p);

/*
 * Block mean-pooling of the keys (each block's representative is the mean of its
 * keys; youleyou.com article, section "MoBA：基于块的混合注意力机制", and its
 * implementation section "PyTorch实现关键要点").
 *   K     [T, Hkv, D] bf16, read once.
 *   Kbar  [num_seqs, MB, Hkv, D] fp32 out: mean over the block's valid tokens,
 *         accumulated in fp32.
 */
MOBA_API moba_status moba_pool_keys(const moba_params* p, const void* K, float* Kbar, void* stream);

/*
 * Parameter-free gate with causal block mask, forced own block and top-k (README
 * bullet "Parameter-less Gating Mechanism"; README FAQ of issue #27: the own block
 * is always taken, top_k-1 more come from strictly earlier blocks, the own block is
 * not a candidate; the article's section "PyTorch实现关键要点": score = query times
 * pooled key, mask future blocks, top-k).
 *   Q     [T, Hq, D] bf16.
 *   Kbar  from moba_pool_keys.
 *   sel   [T, Hq, top_k] int32 out: sel[..,0] = own block i = floor(p/bs);
 *         sel[..,1..m] = the m = min(top_k-1, i) past blocks with the largest
 *         <q, Kbar[b]>, by descending score, ties to the lower block index;
 *         remaining slots -1.
 *         Resolution: scores are fp32 sums of q against Kbar split into bf16 hi + lo
 *         (error up to 2^-18 B, B = |q| max_b |Kbar[b]| over the row's candidates).  With
 *         top_k <= 5 and more than 64 candidate blocks the ranking compares the scores on
 *         a grid of step 2^-18 B / 0.49; scores on the same grid point rank by block
 *         index.  Exact ties always go to the lower block.
 *   workspace: >= moba_workspace_size(p) bytes, 256-byte aligned.
 */
MOBA_API moba_status moba_gate_topk(const moba_params* p, const void* Q, const float* Kbar, int32_t* sel,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Attention over the selected blocks plus online-softmax merge (article section
 * "PyTorch实现关键要点": attention runs separately on the own block, causally, and on
 * the chosen blocks, and the partial results are merged by online softmax; README
 * FAQ of issue #27: the own block goes through the causal varlen path).
 *   Q, K, V  as above; sel from moba_gate_topk (or any caller-made selection that
 *            obeys its contract: slot 0 the own block, then distinct past blocks,
 *            -1 padding at the end).
 *   O    [T, Hq, D] bf16 out;  LSE  [T, Hq] fp32 out.
 *   Scales logits by softmax_scale (default 1/sqrt(D)); fp32 accumulation.
 */
MOBA_API moba_status moba_attn_fwd(const moba_params* p, const void* Q, const void* K, const void* V,
                          const int32_t* sel, void* workspace, size_t workspace_bytes, void* O,
                          float* LSE, void* stream);

/*
 * The whole forward pass: pool, gate, attention.  Kbar and sel may be NULL, in
 * which case they live inside the workspace; when given they receive the
 * intermediate results (same layouts as above).
 */
MOBA_API moba_status moba_fwd(const moba_params* p, const void* Q, const void* K, const void* V,
                     float* Kbar, int32_t* sel, void* workspace, size_t workspace_bytes, void* O,
                     float* LSE, void* stream);

/*
 * Stages of moba_attn_fwd, callable one by one (moba_attn_fwd = route, past, own
 * block + merge, in this order, on one stream; the workspace carries the state).
 *   moba_route:           groups every (token, query head, slot >= 1) by the past
 *                         block it selected (per KV head), MoE-style: counts, scans,
 *                         scatter (article section "PyTorch实现关键要点": organise the
 *                         data after top-k).  Needs top_k >= 2 to do anything.
 *   moba_attn_past:       exact softmax attention of every routed query row over the
 *                         whole selected block (a past block is complete and wholly
 *                         visible); writes normalised partials + LSE into the workspace.
 *   moba_attn_self_merge: causal attention inside each query's own block, then the
 *                         online-softmax merge with the partials; writes O and LSE.
 */
MOBA_API moba_status moba_route(const moba_params* p, const int32_t* sel, void* workspace,
                                size_t workspace_bytes, void* stream);
MOBA_API moba_status moba_attn_past(const moba_params* p, const void* Q, const void* K, const void* V,
                                    void* workspace, size_t workspace_bytes, void* stream);
MOBA_API moba_status moba_attn_self_merge(const moba_params* p, const void* Q, const void* K,
                                          const void* V, const int32_t* sel, void* workspace,
                                          size_t workspace_bytes, void* O, float* LSE, void* stream);

/*
 * The mask-based form of the attention, as a baseline for the efficient path (README section
 * "Implementation Details": moba_naive materialises the block-selection mask and runs masked
 * attention; moba_efficient is the fast form).  Every causal key of the query's sequence is
 * scored, and keys outside the row's selected blocks (from `sel`) get zero weight; the own
 * block is causal.  Same O and LSE as moba_attn_fwd up to rounding, at the cost of dense
 * causal attention (the tensor-core tiles of moba_attn_fwd's own-block stage, extended over
 * the whole prefix).  Needs no workspace.
 *   Q, K, V, sel, O, LSE: as for moba_attn_fwd.
 */
MOBA_API moba_status moba_attn_naive(const moba_params* p, const void* Q, const void* K, const void* V,
                                     const int32_t* sel, void* O, float* LSE, void* stream);

/*
 * Backward pass through the selected blocks, for training (README bullet "Trainable Block
 * Sparse Attention").  The gate has no parameters (README "Parameter-less Gating
 * Mechanism"), so the top-k selection in `sel` is held fixed and the gradients are those
 * of masked softmax attention under MoBA's mask (the selected blocks' keys, causal inside
 * the own block): with P = exp(scale <q, k> - LSE), dP = <dO, v>, Dp = <dO, O> and
 * dS = P (dP - Dp):  dQ = scale sum_j dS k_j,  dK = scale sum_p dS q_p,  dV = sum_p P dO_p
 * (dK and dV summed over the query heads of each KV group).
 *   Q, K, V, sel   the forward's inputs and selection (moba_gate_topk or moba_fwd).
 *   O, LSE         the forward's outputs (O bf16 [T, Hq, D], LSE fp32 [T, Hq]).
 *   dO             [T, Hq, D] bf16, the gradient of the loss with respect to O.
 *   dQ             [T, Hq, D] bf16 out;  dK, dV  [T, Hkv, D] bf16 out.  Every element is
 *                  written (keys that no query attends get 0).
 *   workspace: >= moba_bwd_workspace_size(p) bytes, 256-byte aligned (routing arrays, Dp and
 *   one fp32 dQ partial per routed (token, head, slot)).
 * fp32 accumulation throughout; P and dS enter the tensor cores as bf16.
 */
MOBA_API size_t moba_bwd_workspace_size(const moba_params* p);
MOBA_API moba_status moba_attn_bwd(const moba_params* p, const void* Q, const void* K, const void* V,
                                   const void* O, const float* LSE, const void* dO, const int32_t* sel,
                                   void* workspace, size_t workspace_bytes, void* dQ, void* dK, void* dV,
                                   void* stream);

/*
 * Gated decode: one new query per sequence attends to that sequence's KV cache through the
 * same gate as prefill (README: "Parameter-less Gating Mechanism"; README FAQ of issue #27:
 * own block always taken, top_k-1 more from strictly earlier blocks; README FAQ of issue
 * #30: the released decode path runs full attention instead, which this call does not).
 * The new token is the LAST token of its sequence, at position p = len - 1 in block
 * i = p / bs: its own (possibly partial) block is attended up to p, and the top_k - 1
 * earlier blocks with the largest <q, Kbar[b]> are attended whole; the per-block results
 * are merged by online softmax.  Results equal those of moba_fwd's row for that token.
 *   p     the cache geometry: cu_seqlens over the cached tokens, which INCLUDE the new
 *         token's key and value (every sequence holds >= 1 token, else MOBA_ERR_INVALID_ARG).
 *   Q     [num_seqs, Hq, D] bf16: the new queries.
 *   K, V  [T, Hkv, D] bf16: the caches.
 *   Kbar  [num_seqs, MB, Hkv, D] fp32 pooled keys of the caches (moba_pool_keys once, then
 *         moba_pool_last_block after each append keeps them current; only blocks before
 *         each sequence's last block are read).
 *   sel   [num_seqs, Hq, top_k] int32 out, as for moba_gate_topk; may be NULL.
 *   workspace: >= moba_decode_workspace_size(p) bytes, 256-byte aligned.
 *   O     [num_seqs, Hq, D] bf16 out;  LSE  [num_seqs, Hq] fp32 out.
 */
MOBA_API size_t moba_decode_workspace_size(const moba_params* p);
MOBA_API moba_status moba_decode_fwd(const moba_params* p, const void* Q, const void* K, const void* V,
                                     const float* Kbar, int32_t* sel, void* workspace, size_t workspace_bytes,
                                     void* O, float* LSE, void* stream);

/*
 * Block mean-pooling of each sequence's LAST block only (the one holding its newest token),
 * written into Kbar as moba_pool_keys would write it; every other block of Kbar is left
 * untouched.  Reads at most block_size tokens per sequence: after appending tokens to a KV
 * cache, this keeps Kbar equal to moba_pool_keys of the whole cache as long as each append
 * stays within the sequence's current last block or opens the next one.
 */
MOBA_API moba_status moba_pool_last_block(const moba_params* p, const void* K, float* Kbar, void* stream);

/*
 * moba_gate_topk without a workspace argument.  The MoBA pages have no counterpart: this is
 * an interface convenience, not part of the method.  Same inputs, outputs and results as
 * moba_gate_topk, for callers that cannot allocate device memory: code that enqueues work
 * while a CUDA graph is being captured (cudaMalloc is not allowed then), serving runtimes
 * that forbid allocation after start-up to keep memory use fixed, and host programs that
 * receive raw device pointers but no allocator.  The gate's scratch (the bf16 hi/lo split
 * of Kbar and the pooled keys' squared norms) lives in one device array of
 * MOBA_NOALLOC_MAX_KBAR_ELEMS * 4 bytes (8 MiB) plus 128 KiB that is compiled into the
 * library; every GPU that loads the library holds it until exit.
 *  - Limit: num_seqs * ceil(max_seqlen / block_size) * num_kv_heads * head_dim must not
 *    exceed MOBA_NOALLOC_MAX_KBAR_ELEMS (2^21; a 1M-token sequence with 8 KV heads of
 *    dimension 128 at block size 2048 needs 2^19); larger problems get MOBA_ERR_UNSUPPORTED.
 *  - The first call on each device looks up the array's device address (a CUDA runtime
 *    query, no allocation; concurrent first calls from several host threads are safe); make
 *    that first call before any stream capture begins.  The looked-up address belongs to the
 *    device's primary context and is not valid after cudaDeviceReset on that device.
 *  - All calls share the one array and it keeps the last call's contents; every element a
 *    call reads is written earlier in the same call, so nothing needs clearing.  Calls
 *    whose kernels overlap on the GPU (other streams, other host threads) race on it and
 *    must be serialised by the caller.
 */
#define MOBA_NOALLOC_MAX_KBAR_ELEMS (1u << 21)
MOBA_API moba_status moba_gate_topk_noalloc(const moba_params* p, const void* Q, const float* Kbar,
                                            int32_t* sel, void* stream);

/*
 * The whole forward pass on HOST buffers, with the host<->device copies overlapped with the
 * kernels.  MoBA is independent per KV-head group (each group's queries gate on, and attend
 * to, that group's keys only), so the problem is cut into its Hkv groups: for each group the
 * Q/K/V head slices are copied (2D copies, no host repacking) into a device staging slot,
 * the forward runs on them, and the O/LSE slices are copied back into place.  Group g uses
 * slot g % nstreams and streams[g % nstreams], so copies of one group overlap the kernels
 * and copies of others.  Results equal moba_fwd's.
 *   Q [T, Hq, D], K, V [T, Hkv, D] bf16, O [T, Hq, D] bf16, LSE [T, Hq] fp32: HOST pointers,
 *     page-locked (pinned) for the copies to be asynchronous and to overlap.
 *   staging: DEVICE buffer of moba_host_staging_size(p, nstreams) bytes, 256-byte aligned.
 *   streams: nstreams cudaStream_t handles owned by the caller.
 * Asynchronous: returns once everything is enqueued; synchronise every stream before
 * reading O/LSE or reusing the inputs.  cu_seqlens (host and device) as for moba_fwd.
 */
MOBA_API size_t moba_host_staging_size(const moba_params* p, int nstreams);
MOBA_API moba_status moba_fwd_host(const moba_params* p, const void* Q, const void* K, const void* V, void* O,
                                   float* LSE, void* staging, size_t staging_bytes, void* const* streams,
                                   int nstreams);

/* Kernel launches one moba_fwd enqueues for these params (host only; -1 if invalid). */
MOBA_API int moba_launches_per_forward(const moba_params* p);

/*
 * Device error word of the current device: the tensor-core kernels bound every wait on an
 * mbarrier (about 2 s); a wait that gives up ORs 1 into this word and the kernel returns
 * early instead of hanging.  Reads it synchronously (and zeroes it when `clear` != 0).
 * A non-zero value means the outputs of the affected launches are not valid.
 */
MOBA_API moba_status moba_read_device_error(int32_t* value, int clear);

/*
 * Exercises the failure path of those bounded waits: one thread waits on an mbarrier phase
 * that nothing completes; after the wait limit (about 2 s) it gives up, sets the device error
 * word and returns.  Synchronous.  *device_error receives the word's value (1 when the path
 * works); the word is cleared before and after.
 */
MOBA_API moba_status moba_selftest_bounded_wait(int32_t* device_error);

/* Static description of a status code. */
MOBA_API const char* moba_status_string(int status);

/* Detail of the last error raised on the calling thread ("" if none). */
MOBA_API const char* moba_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* MOBA_H_ */
