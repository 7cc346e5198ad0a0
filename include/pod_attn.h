/*
 * pod_attn.h -- C ABI of libpod_attn.so: one fused attention launch for a
 * hybrid batch of causal prefill chunks and single-token GQA decodes, on an
 * NVIDIA B200 (sm_100a).
 *
 * The operation (POD-Attention: Unlocking Full Prefill-Decode Overlap for
 * Faster LLM Inference, §2.1 "Large Language Model Inference": a hybrid batch
 * holds a prefill chunk and many decodes; §4 "POD-Attention": both run in one
 * fused kernel). For each query row and query head h, with G = H / Hk and
 * KV head g = h / G:
 *
 *     O[row, h, :]  = softmax(q K_g^T / sqrt(d)) V_g     over the visible keys
 *     LSE[row, h]   = ln sum_j exp(q . k_j / sqrt(d))    (natural log, fp32)
 *
 * Visible keys: token t (0-based in its chunk) of a prefill request with
 * `prior` cached tokens sees keys 0 .. prior + t (the chunk's own K/V must
 * already be in the cache at positions prior .. prior + chunk - 1). A decode
 * request with context L sees keys 0 .. L - 1 (its own new K/V already
 * appended). Fusion changes only where and in which order tiles run, never
 * these values (Silicon & Systems digest of the paper, "Virtual CTAs and
 * SM-aware balance").
 *
 * Data types and layouts (all row-major, "NHD"):
 *   Q, O      bf16 [rows, H, d]       (prefill rows = the chunks of all prefill
 *                                      requests back to back, in request order)
 *   LSE       fp32 [rows, H]
 *   K, V      contiguous layout: one bf16 [len, Hk, d] cache per request;
 *             paged layout: one bf16 pool [num_blocks, page_size, Hk, d]
 *             shared by all requests plus an int32 block table whose row r
 *             lists request r's physical block ids in logical order.
 * Supported: d in {64, 128}; H % Hk == 0 with G = H / Hk in 1..8;
 * page_size = 16. Other shapes return POD_EUNSUPPORTED (the caller runs its own
 * separate kernels; there is no CPU fallback -- the digest's
 * "Isolation and predictability" section asks for exactly such a fallback
 * signal).
 *
 * Memory ownership:
 *   - the caller owns every Q, O, LSE, K, V, pool and block-table buffer; all
 *     are DEVICE memory on the context's device, 16-byte aligned;
 *   - the length arrays (chunk_lens, prior_lens, ctx_lens) and the per-request
 *     pointer arrays (k_ptrs, v_ptrs) are HOST memory, read during the call
 *     only;
 *   - the library owns the context, its device workspace (plan, split-KV
 *     partial results, counters, status word), a pinned host plan ring, and an
 *     internal stream and events. All of it is allocated in pod_attn_create and
 *     released in pod_attn_destroy: the per-call entry points allocate nothing.
 *
 * Calls are asynchronous on the given stream (a cudaStream_t passed as void*;
 * NULL = the legacy default stream) and never synchronise the device. A
 * context must not be used from two streams at once.
 *
 * Errors: host-detectable problems return a negative pod_status BEFORE
 * anything is enqueued. Device-side problems (a bounded wait that ran out)
 * set a sticky status word that pod_attn_status() and pod_attn_destroy()
 * report.
 *
 * Slots of a partially filled last page (paged layout) must hold finite
 * values (e.g. zeros): they are read by whole-page copies and multiplied by a
 * zero softmax weight.
 */
#ifndef POD_ATTN_H
#define POD_ATTN_H

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define POD_API __attribute__((visibility("default")))
#else
#define POD_API
#endif

typedef struct pod_attn_ctx pod_attn_ctx; /* opaque, library-owned */

typedef enum {
  POD_OK = 0,
  POD_EINVAL = -1,        /* NULL pointer, negative length, H % Hk != 0, ... */
  POD_EUNSUPPORTED = -2,  /* head_dim not 64/128, G > 8, page_size != 16     */
  POD_ENOMEM = -3,        /* workspace allocation failed (create only)      */
  POD_ECUDA = -4,         /* a CUDA runtime/driver call failed              */
  POD_ETIMEOUT = -5,      /* device: a bounded wait ran out (sticky)        */
  POD_ECAPACITY = -6      /* sizes exceed the caps given at create          */
} pod_status;

typedef enum { POD_KV_CONTIGUOUS = 0, POD_KV_PAGED = 1 } pod_kv_layout;

/* How pod_attn_hybrid runs the batch.
 * FUSED: one persistent launch, one CTA per SM; the CTA reads its SM id and
 *   takes prefill or decode work units from per-SM tickets (POD-Attention §4.1
 *   "SM-aware CTA Scheduling", §4.4 persistent-thread form, §5.4.2 role
 *   allocation) while two of its warps stream decode units throughout.
 * SERIAL: the prefill-only launch, then the decode launch and the merge
 *   launch, on the caller's stream (the paper's FA_Serial baseline, §2.1/§3).
 * TWO_STREAM: prefill on the caller's stream, decode + merge on an internal
 *   stream, joined back with events (the paper's FA_Streams baseline, §3.2).
 * The decode decomposition is the same in all three modes. The prefill KV
 * split count may differ: a FUSED call that also carries decodes leaves the
 * prefill unsplit, the other modes split it when that shortens the prefill
 * launch. Split partials are merged in split order, so on a common plan the
 * modes' outputs are bitwise identical, and otherwise they differ only by the
 * rounding of the merge. */
typedef enum { POD_MODE_FUSED = 0, POD_MODE_SERIAL = 1, POD_MODE_TWO_STREAM = 2 } pod_mode;

/* Flags for pod_attn_config.flags */
#define POD_FLAG_STATS 0x1u               /* count claimed units per SM and role */
#define POD_FLAG_TEST_FORCE_TIMEOUT 0x2u  /* test only: one CTA waits on a flag that
                                             nothing sets, with a ~1 ms budget, then
                                             records POD_ETIMEOUT and carries on */

typedef struct {
  int num_qo_heads;        /* H                                               */
  int num_kv_heads;        /* Hk; H % Hk == 0                                 */
  int head_dim;            /* d: 64 or 128                                    */
  int kv_layout;           /* pod_kv_layout                                   */
  int page_size;           /* 16 when paged, ignored otherwise                */
  int max_prefill_reqs;    /* <= 16                                           */
  int max_prefill_tokens;  /* cap on sum of chunk lengths per call            */
  int max_decode_reqs;     /* cap on decodes per call                         */
  long long max_kv_tokens; /* cap on any one request's prior + chunk or ctx   */
  int device;              /* CUDA device ordinal the context lives on        */
  unsigned flags;          /* POD_FLAG_*                                      */
} pod_attn_config;

/* Prefill requests of one call (request p owns Q/O rows
 * [sum_{i<p} chunk_i, sum_{i<=p} chunk_i)). */
typedef struct {
  int num_reqs;                 /* 0 .. max_prefill_reqs                        */
  const int* chunk_lens;        /* host [num_reqs], each >= 0 (0 = no-op)      */
  const int* prior_lens;        /* host [num_reqs], each >= 0                  */
  const void* q;                /* device bf16 [sum chunk, H, d]               */
  void* o;                      /* device bf16 [sum chunk, H, d] (written)     */
  float* lse;                   /* device fp32 [sum chunk, H] (written)        */
  const void* const* k_ptrs;    /* contiguous: host array of device pointers,  */
  const void* const* v_ptrs;    /*   request p -> bf16 [prior+chunk, Hk, d]    */
  const void* k_pool;           /* paged: device bf16 [pool_blocks, 16, Hk, d] */
  const void* v_pool;
  const int* block_table;       /* paged: device int32 [num_reqs, stride]      */
  int block_table_stride;       /* entries per block-table row                 */
  long long pool_blocks;        /* paged: number of blocks in the pool         */
} pod_prefill_args;

/* Decode requests of one call (request r owns Q/O row r). */
typedef struct {
  int num_reqs;                 /* 0 .. max_decode_reqs                         */
  const int* ctx_lens;          /* host [num_reqs], each >= 1                  */
  const void* q;                /* device bf16 [num_reqs, H, d]                */
  void* o;                      /* device bf16 [num_reqs, H, d] (written)      */
  float* lse;                   /* device fp32 [num_reqs, H] (written)         */
  const void* const* k_ptrs;    /* contiguous: host array of device pointers,  */
  const void* const* v_ptrs;    /*   request r -> bf16 [ctx, Hk, d]            */
  const void* k_pool;           /* paged: device bf16 [pool_blocks, 16, Hk, d] */
  const void* v_pool;
  const int* block_table;       /* paged: device int32 [num_reqs, stride]      */
  int block_table_stride;
  long long pool_blocks;
} pod_decode_args;

/* What the planner decided for the last call (for tests and the benchmark). */
typedef struct {
  int num_sms;               /* SMs on the device                             */
  int slots_per_sm;          /* persistent CTAs per SM in the fused launch    */
  int prefill_units;         /* (request, pair of 128-row tiles, split) units */
  int prefill_split;         /* KV splits per prefill tile (max over reqs)    */
  int decode_units;          /* (request, KV head, KV split) units            */
  int decode_split_len;      /* keys per decode split                         */
  int ratio_num, ratio_den;  /* prefill share of claims per SM               */
  long long plan_bytes;      /* bytes copied host -> device for the plan      */
  int prefill_sm_cap;        /* fused CTAs that take prefill work first       */
  int pair_clusters;         /* prefill on CTA pairs: clusters of two CTAs;
                                0 when each prefill unit runs on one SM       */
} pod_plan_info;

/* Per-SM role counts gathered with POD_FLAG_STATS (the "virtual CTA mix"). */
typedef struct {
  int num_sms;
  long long prefill_claims;  /* total prefill units claimed                   */
  long long decode_claims;   /* total decode claims (each = one CTA's batch)  */
  int sms_with_both;         /* SMs that ran both roles in the last call      */
} pod_stats;

/* Validates cfg, allocates the workspace on cfg->device. *out is set on
 * success only. Returns POD_OK, POD_EINVAL, POD_EUNSUPPORTED, POD_ENOMEM or
 * POD_ECUDA.
 * Follows: the fused kernel is sized for whichever phase needs more shared
 * memory (POD-Attention summary §4.3 "Implementing CTA-parallel Fusion"), and
 * its split prefill and virtual decode units write partial results that a
 * merge combines (§4.2.3 "Virtual Decode CTAs"): every buffer for those is
 * allocated here, once. The create-time caps bound what one call admits
 * (Silicon & Systems digest, "Isolation and predictability"). */
POD_API int pod_attn_create(pod_attn_ctx** out, const pod_attn_config* cfg);

/* One hybrid batch. Either argument may be NULL or have num_reqs == 0.
 * mode is a pod_mode. stream is a cudaStream_t.
 * Follows: a hybrid batch of prefill chunks and decodes (POD-Attention summary
 * §2.1 "Large Language Model (LLM) Inference") computed by one fused kernel
 * (§4 "POD-Attention", §4.4 persistent form), or by the separate-kernel
 * baselines FA_Serial and FA_Streams (§3.2 "Analysis of Readily Available
 * Methods"). Returns POD_OK, POD_EINVAL, POD_ECAPACITY or POD_ECUDA before
 * or at enqueue time; device problems go to the status word. */
POD_API int pod_attn_hybrid(pod_attn_ctx* ctx, const pod_prefill_args* prefill,
                    const pod_decode_args* decode, int mode, void* stream);

/* Prefill requests alone (the persistent launch with no decode work): the
 * compute-bound phase of the summary's §2.1, as the serial baseline runs it
 * (§3.2). Errors as for pod_attn_hybrid. */
POD_API int pod_attn_prefill_only(pod_attn_ctx* ctx, const pod_prefill_args* prefill, void* stream);

/* Decode requests alone (split-KV decode launch + LSE merge launch): the
 * memory-bound phase of the summary's §2.1, in one-warp units with a
 * 16-key tile (§4.2.1 "Tile Sizes", §4.2.3 "Virtual Decode CTAs"). Errors as
 * for pod_attn_hybrid. */
POD_API int pod_attn_decode_only(pod_attn_ctx* ctx, const pod_decode_args* decode, void* stream);

/* Synchronises `stream`, then returns and clears the sticky device status
 * (POD_OK or POD_ETIMEOUT), or POD_ECUDA if the synchronisation failed.
 * (No counterpart in the pages: the failure signal of the digest's
 * "Isolation and predictability".) */
POD_API int pod_attn_status(pod_attn_ctx* ctx, void* stream);

/* Planner decisions of the last call: split counts, the prefill tile, the
 * role ratio (the summary's §4.2.2, §4.2.3 and §5.4). POD_EINVAL on NULL. */
POD_API int pod_attn_last_plan(const pod_attn_ctx* ctx, pod_plan_info* out);

/* Synchronises `stream` and reads the per-SM role counters of the last call
 * (requires POD_FLAG_STATS at create, else POD_EINVAL): which SMs ran both
 * prefill and decode work (the co-location of the summary's §4.1). */
POD_API int pod_attn_get_stats(pod_attn_ctx* ctx, void* stream, pod_stats* out);

/* Synchronises the device, reads the sticky status, frees everything.
 * Returns that status (POD_OK or POD_ETIMEOUT) or POD_ECUDA. NULL is a no-op.
 * (Resource release; no counterpart in the pages.) */
POD_API int pod_attn_destroy(pod_attn_ctx* ctx);

/* ---------------------------------------------------------------------------
 * Decode attention that allocates nothing (no counterpart in the paper: it
 * is a deployment convenience of this library).
 *
 * For callers that cannot allocate device memory when they call attention:
 * an inference engine that reserves nearly all HBM for its KV-cache pool up
 * front, a plugin that may only use the buffers its host framework gives it,
 * or a loop that cannot afford cudaMalloc's implicit synchronisation. A
 * pod_attn context allocates its workspace at create time, so this entry
 * point needs none: it runs the same split-KV decode and LSE merge kernels as
 * pod_attn_decode_only, with their plan tables, counters and partial results
 * in a fixed device array inside the library (about 16.5 MB, present on
 * every GPU that loads the library until the process exits). It calls no
 * cudaMalloc, cudaFree or other allocating routine.
 *
 * Arguments: head counts and head_dim as in pod_attn_config, kv_layout a
 * pod_kv_layout, `args` exactly as for pod_attn_decode_only (caller-owned
 * device tensors, host length and pointer arrays), `stream` a cudaStream_t.
 * The call runs on the calling thread's current device.
 *
 * Limits (POD_ECAPACITY beyond them, checked before anything is enqueued):
 * num_reqs <= POD_STATIC_MAX_DECODE_REQS, num_kv_heads <=
 * POD_STATIC_MAX_KV_HEADS, num_reqs * num_kv_heads <= POD_STATIC_MAX_UNITS.
 * Other errors as for pod_attn_decode_only.
 *
 * The first call on a device resolves the array's device address and sets
 * the kernels' shared-memory limits for that device; make that first call
 * before any stream capture. Every call reuses the same array and leaves its
 * contents behind (each call re-initialises what must start at zero), so
 * calls that overlap on the GPU -- on different streams or from different
 * host threads -- race on it and must not be issued. The copy of the small
 * per-call plan comes from one pageable host buffer that the next call
 * overwrites, so the call does not return before the stream has reached it,
 * and while `stream` is being captured the call returns POD_EUNSUPPORTED
 * without enqueuing anything. If a device-side wait runs out, the call has
 * no context to hold a status word: it writes NaN to every O and LSE element
 * of the batch instead of a result.
 * ------------------------------------------------------------------------- */
#define POD_STATIC_MAX_DECODE_REQS 512
#define POD_STATIC_MAX_KV_HEADS 16
#define POD_STATIC_MAX_UNITS 4096
POD_API int pod_attn_decode_static(int num_qo_heads, int num_kv_heads, int head_dim,
                                   int kv_layout, const pod_decode_args* args, void* stream);

/* Static string for a pod_status value. */
POD_API const char* pod_attn_strerror(int status);

#ifdef __cplusplus
}
#endif
#endif /* POD_ATTN_H */
