/*
 * fb.h — C ABI of libfb, the B200 (sm_100a) FlashBlock attention step.
 *
 * FlashBlock ("FlashBlock: Attention Caching for Efficient Long-Context Block
 * Diffusion", technical summary section "Mécanisme Central") splits the
 * attention of the current block's queries into a block-external part over the
 * prefix KV cache (A_out, L_out = log Z_out) and a block-internal part over the
 * block's own keys (A_in, L_in), and recombines them with the log-space merge
 *     m = max(L_out, L_in),
 *     A = (e^{L_out-m} A_out + e^{L_in-m} A_in) / (e^{L_out-m} + e^{L_in-m}).
 * A_out/L_out are cached across diffusion steps and reused while fewer than tau
 * tokens changed, and for video only in heads whose similarity exceeds gamma
 * (section "Stratégies de Réutilisation Adaptatives").
 *
 * Conventions for every call
 * --------------------------
 * - Tensors are caller-owned device memory.  Q/O are [B, Hq, Nb, D], K_in/V_in
 *   [B, Hkv, Nb, D], K_p/V_p [B, Hkv, kp_capacity, D]; the head dimension is
 *   contiguous and the batch, head and token strides (in elements) are given in
 *   the descriptor.  V shares its K's strides.  Query head h reads KV head
 *   h / (Hq / Hkv).
 * - A "part" (A, L) is fp32 and packed: A [B, Hq, Nb, D] and L [B, Hq, Nb],
 *   A normalised (a softmax average of values) and L = log Z in natural log.
 *   An empty key set is (A, L) = (0, -inf).
 * - Requirements: D in {64, 128}; Hq % Hkv == 0; every pointer 16-byte
 *   aligned; every token stride times the element size a multiple of 16 bytes.
 * - Every call checks its arguments on the host first; a failed check returns
 *   an error and launches nothing.  Work is queued on `stream` and the call
 *   returns without synchronising; no call allocates device memory.  Buffers
 *   must stay valid until the queued work has finished.
 * - Kernels that wait on barriers bound each wait (about 2 s by default); on
 *   expiry they record FB_ETIMEOUT in a per-device status word and return
 *   without touching their outputs further.  fb_get_device_status() reads it.
 *   The word's device address is looked up at the first launch on each
 *   device: make one call on a device before capturing its work in a CUDA
 *   graph.  The library is not usable after a cudaDeviceReset in the same
 *   process (cached device addresses and function attributes go stale).
 * - Handles are not thread-safe.
 */
#ifndef FB_H
#define FB_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fb_status {
  FB_OK = 0,
  FB_EINVAL = 1,        /* null pointer, bad size, shape or count */
  FB_EALIGN = 2,        /* pointer or stride breaks the 16-byte rule */
  FB_EDTYPE = 3,        /* unknown or unsupported dtype combination */
  FB_EUNSUPPORTED = 4,  /* valid but not implemented (e.g. D = 96) */
  FB_ESTATE = 5,        /* handle state forbids the call */
  FB_ECUDA = 6,         /* a CUDA runtime call failed (launch, memset, copy) */
  FB_ETIMEOUT = 7,      /* a kernel's bounded wait expired (device status) */
  FB_ENOSPACE = 8       /* the workspace given is smaller than required */
} fb_status;

typedef enum fb_dtype { FB_F32 = 0, FB_BF16 = 1 } fb_dtype;

#define FB_MAX_PARTS 8       /* parts merged by fb_merge / fb_attn_inblock */
#define FB_TAU_OFF INT32_MAX /* tau value that turns the tau gate off */

typedef struct fb_attn_desc {
  int32_t B, Hq, Hkv, D, Nb;  /* batch, query heads, KV heads, head dim, block length */
  int32_t in_dtype;           /* fb_dtype of Q, K_in, V_in, K_p, V_p */
  int32_t out_dtype;          /* fb_dtype of O */
  float scale;                /* softmax scale; 0 selects 1/sqrt(D) */
  int64_t kp_capacity;        /* token rows allocated per (b, kv head) in K_p/V_p */
  int64_t q_strides[3];       /* Q: batch, head, token strides in elements */
  int64_t kin_strides[3];     /* K_in and V_in */
  int64_t kp_strides[3];      /* K_p and V_p */
  int64_t o_strides[3];       /* O */
} fb_attn_desc;

/* Human-readable name of a status code (static string). */
const char* fb_status_string(fb_status s);

/* Library ABI version: (major << 16) | minor. */
int32_t fb_version(void);

/* ---------------------------------------------------------------------------
 * Block-external attention (summary, "Mécanisme Central": A_out over J_out
 * with L_out = log Z_out; "Stratégies de Réutilisation Adaptatives", sparse
 * bullet: unselected keys form the block-external set).
 *
 * Dense (sel == NULL): (a_out, l_out) = attention of Q over prefix rows
 *   [0, prefix_len) of K_p/V_p.  prefix_len == 0 gives (0, -inf).
 * Sparse (sel != NULL): sel is device int32 [B, Hq, sel_k], each row strictly
 *   ascending positions in [0, prefix_len).  (a_out, l_out) covers the selected
 *   keys S; when a_res != NULL, (a_res, l_res) covers the rest, prefix minus S.
 * ws/ws_bytes: device scratch of at least fb_outblock_workspace_bytes() bytes
 *   (split-KV partial results); its contents need no initialisation.
 * Errors: FB_EINVAL (null tensors, prefix_len < 0 or > kp_capacity, sel_k < 0
 *   or > prefix_len), FB_EALIGN, FB_EDTYPE, FB_EUNSUPPORTED, FB_ENOSPACE,
 *   FB_ECUDA.
 * ------------------------------------------------------------------------- */
fb_status fb_outblock_workspace_bytes(const fb_attn_desc* d, int64_t prefix_len,
                                      int32_t sel_k, size_t* bytes);
fb_status fb_attn_outblock(const fb_attn_desc* d, const void* q, const void* kp,
                           const void* vp, int64_t prefix_len,
                           const int32_t* sel, int32_t sel_k,
                           float* a_out, float* l_out,
                           float* a_res, float* l_res,
                           void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Dense block-external attention for callers that cannot allocate.  The pages
 * have no counterpart: this is a library service, not part of the method.
 *
 * Same arguments and result as fb_attn_outblock with sel == NULL, but without
 * a workspace argument: the split-KV partial results go to a fixed array of
 * FB_NOALLOC_SCRATCH_BYTES inside the library.  It is for callers that cannot
 * call cudaMalloc or pass scratch at call time. Examples: code whose host
 * framework owns the whole device pool, plug-ins limited to memory their host
 * hands them, and services that must not allocate while serving.
 * - Every GPU on which the library is loaded keeps the array until the
 *   process exits.
 * - The first call on a device looks up the array's device address (with
 *   that device current) and caches it.  Make that first call before any
 *   stream capture.  The cached address does not survive a cudaDeviceReset
 *   in the same process: do not call the library after one.
 * - All calls share the array, and it keeps the last call's contents; this
 *   call overwrites everything it reads, so it needs no clearing.  Calls whose
 *   work overlaps on the GPU (unordered streams) race on it.
 * - Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * Errors: as fb_attn_outblock; FB_ENOSPACE when the call would need more than
 *   FB_NOALLOC_SCRATCH_BYTES of scratch (fb_outblock_workspace_bytes with
 *   sel_k = 0 gives the need).
 * ------------------------------------------------------------------------- */
#define FB_NOALLOC_SCRATCH_BYTES (64u << 20)
fb_status fb_attn_outblock_noalloc(const fb_attn_desc* d, const void* q, const void* kp,
                                   const void* vp, int64_t prefix_len,
                                   float* a_out, float* l_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Selection of the sparse keys by attention mass (summary, "Stratégies de
 * Réutilisation Adaptatives", sparse bullet: FlashBlock caches the residual of
 * the keys a sparse method leaves out; "Résultats Expérimentaux": SparseD at
 * 20-40 % density).  The pages do not give the sparse method's rule; this
 * call keeps, per (b, query head), the k prefix keys of largest
 *     mass_j = sum_i exp(scale q_i . k_j - L_out,i)
 * (the softmax probability over the prefix that key j receives from the
 * block's queries, summed over them), ties to the lower index.  Call it once
 * per block with the block's first queries and pass sel_out to that block's
 * fb_step calls.
 * sel_out: device int32 [B, Hq, k], written ascending (may be NULL when
 *   k == 0).  mass_out: optional
 *   device fp32 [B, Hq, prefix_len] that receives the masses (else they stay
 *   in the workspace).  ws: at least fb_select_workspace_bytes() bytes.
 * Requires bf16 inputs, D = 128, Nb in {16, 32} and (Hq / Hkv) * Nb <= 128
 * (FB_EUNSUPPORTED otherwise).  The masses are fp32 sums in a fixed order, so
 * a selection is the same on every run; near-tied keys at the k-th place may
 * rank differently from an exact computation.
 * Errors: FB_EINVAL (k outside [0, prefix_len], prefix_len < 1), FB_EALIGN,
 *   FB_EUNSUPPORTED, FB_ENOSPACE, FB_ECUDA.
 * ------------------------------------------------------------------------- */
fb_status fb_select_workspace_bytes(const fb_attn_desc* d, int64_t prefix_len, size_t* bytes);
fb_status fb_select_mass(const fb_attn_desc* d, const void* q, const void* kp, const void* vp, int64_t prefix_len,
                         int32_t k, int32_t* sel_out, float* mass_out, void* ws, size_t ws_bytes,
                         cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Block-internal attention fused with the log-space merge (summary,
 * "Mécanisme Central": A_in over J_in, merged with the block-external parts).
 *
 * Attention of Q over all Nb keys of K_in/V_in (bidirectional), merged with
 * `nparts` (0..FB_MAX_PARTS-1) fp32 parts given as host arrays of device
 * pointers a_parts[i], l_parts[i] (for instance the cached A_out/L_out).
 * Writes O (out_dtype, o_strides) and, if lse != NULL, the merged natural-log
 * normaliser, fp32 packed [B, Hq, Nb].  The prefix K/V are never read.
 * Errors: FB_EINVAL, FB_EALIGN, FB_EDTYPE, FB_EUNSUPPORTED, FB_ECUDA.
 * ------------------------------------------------------------------------- */
fb_status fb_attn_inblock(const fb_attn_desc* d, const void* q, const void* kin,
                          const void* vin, int32_t nparts,
                          const float* const* a_parts, const float* const* l_parts,
                          void* o, float* lse, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Standalone N-way log-space merge (summary, "Mécanisme Central", merge
 * equation, applied to 1..FB_MAX_PARTS parts over disjoint key sets):
 *   m = max_p L_p, w_p = e^{L_p - m}, O = sum w_p A_p / sum w_p,
 *   LSE = m + log sum w_p; rows whose parts are all empty give (0, -inf).
 * a_parts/l_parts: host arrays of nparts device pointers (packed parts).
 * O: out_dtype with o_strides; lse: fp32 packed, may be NULL.
 * Errors: FB_EINVAL, FB_EALIGN, FB_EDTYPE, FB_ECUDA.
 * ------------------------------------------------------------------------- */
fb_status fb_merge(const fb_attn_desc* d, int32_t nparts,
                   const float* const* a_parts, const float* const* l_parts,
                   void* o, float* lse, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * KV cache append (summary, section 1 "Énoncé du Problème"; abstract: block
 * diffusion grows the KV cache block by block).  Copies K_in/V_in into
 * K_p/V_p rows [prefix_len, prefix_len + Nb) of every (b, kv head).
 * Errors: FB_EINVAL (prefix_len + Nb > kp_capacity), FB_EALIGN, FB_ECUDA.
 * ------------------------------------------------------------------------- */
fb_status fb_kv_append(const fb_attn_desc* d, void* kp, void* vp,
                       int64_t prefix_len, const void* kin, const void* vin,
                       cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Cache handle and the FlashBlock step (summary, "Mécanisme Central" and
 * "Stratégies de Réutilisation Adaptatives").
 *
 * The handle keeps, in caller-owned device memory `dev_mem`, the cached
 * block-external part per (b, h) (the prefix part, or for sparse steps the
 * residual over the unselected keys), the per-head similarities and reuse mask
 * of the gamma gate, and scratch for split-KV partial results.  The handle
 * itself is host memory holding sizes, pointers and the host-side validity.
 *
 * flags: FB_CACHE_SPARSE enables sparse steps (sel != NULL), FB_CACHE_GAMMA
 *   enables the gamma gate, FB_CACHE_ACTIVE steps over active-query subsets
 *   (active != NULL).  max_prefix / max_sel_k bound later calls.
 * fb_cache_create() zeroes its bookkeeping with cudaMemsetAsync on `stream`.
 * fb_cache_begin_block() marks the cache invalid, so the next step is full.
 * ------------------------------------------------------------------------- */
typedef struct fb_cache* fb_cache_t;

enum { FB_CACHE_SPARSE = 1, FB_CACHE_GAMMA = 2, FB_CACHE_ACTIVE = 4 };

fb_status fb_cache_workspace_bytes(const fb_attn_desc* d, int32_t flags,
                                   int64_t max_prefix, int32_t max_sel_k,
                                   size_t* bytes);
fb_status fb_cache_create(const fb_attn_desc* d, int32_t flags, int64_t max_prefix,
                          int32_t max_sel_k, void* dev_mem, size_t bytes,
                          cudaStream_t stream, fb_cache_t* out);
fb_status fb_cache_destroy(fb_cache_t c);
fb_status fb_cache_begin_block(fb_cache_t c, cudaStream_t stream);

typedef struct fb_step_args {
  const void* q;          /* [B, Hq, Nb, D] this step's block queries */
  const void* kin;        /* [B, Hkv, Nb, D] this step's block keys */
  const void* vin;        /* [B, Hkv, Nb, D] this step's block values */
  const void* kp;         /* prefix cache keys   [B, Hkv, kp_capacity, D] */
  const void* vp;         /* prefix cache values [B, Hkv, kp_capacity, D] */
  int64_t prefix_len;     /* valid prefix rows (<= max_prefix) */
  int32_t M;              /* tokens updated since the previous step */
  int32_t tau;            /* reuse only if M < tau; FB_TAU_OFF: gate off */
  const float* gamma;     /* device fp32 [Hq] thresholds, or NULL: gate off */
  const int32_t* sel;     /* device int32 [B, Hq, sel_k] ascending, or NULL */
  int32_t sel_k;
  void* o;                /* output [B, Hq, Nb, D] (out_dtype, o_strides) */
  float* lse;             /* output fp32 [B, Hq, Nb] natural log, or NULL */
  int8_t* reuse_out;      /* output int8 [B, Hq]: 1 where the cache was used, or NULL */
  float* sim_out;         /* output fp32 [B, Hq]: similarity after the step (NaN:
                             not yet defined), or NULL */
  const int32_t* active;  /* device int32 [B, n_active]: the block positions still
                             active (unlocked), ascending; NULL: all Nb positions */
  int32_t n_active;       /* 1..Nb when active != NULL */
} fb_step_args;

/* One diffusion step of one attention layer under the reuse policy:
 *   reuse(b, h) = cache valid && M < tau && (gamma off || sim(b, h) > gamma[h]).
 * The cache is valid from the first step after fb_cache_begin_block on, and
 * only for the block-external key set it was computed over: a step whose
 * prefix_len, or sparse selection size sel_k (or dense/sparse kind), differs
 * from the last step's starts over as at a new block (full step, similarities
 * undefined).  A caller that changes the selection's contents but not its size
 * must call fb_cache_begin_block itself.
 * Heads that do not reuse recompute the block-external part over the prefix
 * (or the residual, for sparse steps), refresh the cache and, with the gamma
 * gate on and the cache valid, refresh sim(b, h) = cosine of the fresh and the
 * cached part flattened over [Nb, D].  A reusing head keeps its cache and
 * similarity.  Every head then merges the block-external part (for sparse
 * steps: the selected keys' fresh part and the cached residual) with fresh
 * block-internal attention.  The tau decision is taken on the host; the gamma
 * decision on the device, from the similarity of an earlier step.
 * Errors: FB_EINVAL, FB_EALIGN, FB_EDTYPE, FB_EUNSUPPORTED, FB_ESTATE (sparse
 *   step on a handle without FB_CACHE_SPARSE, gamma without FB_CACHE_GAMMA),
 *   FB_ECUDA. */
fb_status fb_step(fb_cache_t c, const fb_step_args* a, cudaStream_t stream);

/* Active-query subsets (SureLock page, "Principes de Fonctionnement", items 2
 * and 3): with a->active set, only the n_active listed positions of the block
 * query.  Their block-external part is recomputed on a full step (the cache
 * rows of the other positions are left as they are), they attend to all Nb
 * keys of the block (locked positions' K/V stay in K_in/V_in), and only their
 * rows of O and LSE are written: a locked position keeps whatever the caller's
 * O and LSE hold (its output of an earlier step).  Locking must be monotone
 * within a block (a position locked once stays locked until
 * fb_cache_begin_block), so every active position's cache row dates from the
 * last full step; the library does not check this.  Requires FB_CACHE_ACTIVE,
 * bf16 inputs, D = 128, Nb <= 64, no selection and no gamma gate
 * (FB_EUNSUPPORTED otherwise).  A listed position outside [0, Nb) is skipped
 * and reported as FB_EINVAL in the device status word. */

/* Host-side decision of the last fb_step: *recomputed = 1 when the tau gate
 * (or an invalid cache) forced a full step. */
fb_status fb_cache_last_step(fb_cache_t c, int32_t* recomputed);

/* Synchronises `stream`, then reads and clears this device's status word:
 * *device_status = FB_OK or the first error a kernel recorded (FB_ETIMEOUT). */
fb_status fb_get_device_status(cudaStream_t stream, fb_status* device_status);

/* ---------------------------------------------------------------------------
 * Profiling hook (no counterpart on the pages; used by the benchmark).  While
 * enabled, every kernel launch of the library is bracketed by CUDA events
 * recorded on its launching stream, and the library adds up, per kernel kind,
 * the launches, their event-timed duration and their algorithmic bytes (the
 * bytes the step must move at least: inputs read once, outputs written once;
 * split-KV partials and re-reads do not count).
 * Kinds: 0 block-external (prefix) attention, 1 block-internal attention with
 * the fused merge, 2 merge / gamma update / append / bitmap.
 * fb_profile_read synchronises on every recorded event; with reset != 0 it
 * then clears the totals.  arrays have FB_PROFILE_KINDS entries.
 * ------------------------------------------------------------------------- */
#define FB_PROFILE_KINDS 3
fb_status fb_profile_enable(int32_t on);
fb_status fb_profile_read(int32_t reset, int64_t* launches, double* total_ms, double* alg_bytes);

/* Test hook: which kernel runs dense block-external passes: 0 automatic (the
 * tcgen05 kernel where the shape and strides allow it), 1 the generic
 * mma.sync / FFMA kernel only, 2 the tcgen05 kernel whenever it applies,
 * 3 as 2 but its key splits always go through a separate merge instead of
 * the in-kernel cluster reduction, 4 as 2 with the split planner charging
 * nothing for the cluster reduction (so it is taken wherever it saves
 * waves or parts). */
fb_status fb_debug_set_prefix_kernel(int32_t which);

/* Test hook: the bound of every barrier wait in later launches, in
 * nanoseconds (default 2e9).  0 makes any wait that is not already satisfied
 * expire at once.  Affects only the calling process. */
fb_status fb_debug_set_wait_limit_ns(uint64_t ns);

/* Test hook: when on, each tcgen05 prefix/in-block kernel and each small
 * in-block kernel launched afterwards first waits on a barrier that nothing
 * completes, so that wait runs out after the configured limit and the launch
 * records FB_ETIMEOUT (every CTA still drains its own copies and MMAs before
 * it returns).  Off by default.  Affects only the calling process. */
fb_status fb_debug_set_stall(int32_t on);

/* Tuning hook: which kernel runs block-internal passes: 0 (default)
 * automatic (the small mma.sync kernel for blocks of up to 64 keys, the
 * paired tcgen05 kernel above), 1 the paired tcgen05 kernel wherever it
 * applies (two or more 128-row query tiles per KV head).  Affects only the
 * calling process. */
fb_status fb_debug_set_inblock_kernel(int32_t which);

/* Tuning hook: how the small-block in-block kernel loads its rows: 0
 * (default) 16-byte cp.async chunks from every thread, 1 one bulk copy per
 * row.  Affects only the calling process. */
fb_status fb_debug_set_inblock_loads(int32_t bulk);

/* Tuning hook: how the small-block in-block kernel (blocks of up to 64 keys)
 * splits its work: 0 (default) automatic, 16, 32 or 64 one warp per 16 query
 * rows with CTAs of that many rows of one KV head, 1 the split-warp kernel
 * (CTAs of 16 rows whose four warps share S and split the head dimension).
 * Any other value is FB_EINVAL.  Affects only the calling process. */
fb_status fb_debug_set_inblock_rows(int32_t rows);

/* Tuning hook: 1 (default) launches every kernel with programmatic dependent
 * launch allowed, so a kernel's launch overlaps the tail of the one before it
 * in the stream (each kernel waits for its predecessors before it touches
 * global memory); 0 launches them in plain stream order.  Affects only the
 * calling process. */
fb_status fb_debug_set_pdl(int32_t on);

#ifdef __cplusplus
}
#endif
#endif /* FB_H */
