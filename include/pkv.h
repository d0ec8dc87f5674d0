/*
 * pkv.h - C ABI of the B200 (sm_100a) paged-KV attention library (libpkv.so).
 *
 * Batched attention over a paged KV cache: causal or full GQA prefill, the
 * memory-bound decode case (one query per request) and the absorbed-MLA
 * variant. Every call writes O (bf16) and a base-2 log-sum-exp per
 * (token, head) (fp32).
 *
 * Where each operation is defined
 *   - Page table kv_indptr / kv_indices / kv_last_page_len and the ragged query
 *     layout [total_q, num_qo_heads, head_dim] cut by qo_indptr:
 *     flashinfer-trace discussion #15, "Notes on fa3_gqa_prefill_v1";
 *     FlashInfer 0.7.4 documentation, "KV-Cache Layout in FlashInfer"
 *     ("Layout: NHD/HND", "Ragged Tensor", "Page Table Layout").
 *   - page_size as the column width of one sparse block, page_size = 1 being
 *     vector sparsity: FlashInfer 0.2 release, "FlashAttention-3 template with
 *     block/vector sparsity".
 *   - Base-2 LSE: discussion #15, same notes (natural-log LSE / ln 2).
 *   - plan / run split, plan taking host arrays and copying its schedule to
 *     the device without blocking: FlashInfer 0.2 release, "Faster plan function".
 *   - Split-KV (the disable_split_kv knob) and merging attention states:
 *     discussion #15, "Tunable Solutions and their Implementation Configs";
 *     documentation, "Attention States and Recursive Attention",
 *     "Merge Attention States".
 *   - MLA with matrix absorption, scores q_nope.ckv + q_pe.kpe, output P.ckv:
 *     FlashInfer 0.2 release, "Fused MLA decode kernel"; definition
 *     mla_paged_prefill_causal_h16_ckv512_kpe64_ps1 (discussion #15).
 *
 * Semantics (readings where the pages are silent)
 *   - O = softmax(sm_scale * Q K^T) V per (token, qo head); qo head h reads kv
 *     head h / (num_qo_heads / num_kv_heads).
 *   - Causal masking is bottom-right aligned: query i of a request with qo_len
 *     queries and kv_len keys sees key j iff j <= i + kv_len - qo_len.
 *   - A row that sees no key gets O = 0 and LSE = -inf.
 *   - lse[t, h] = log2(sum_j exp(sm_scale * q.k_j)).
 *
 * Layouts (all row-major, contiguous, device memory unless marked HOST)
 *   q        bf16 [total_q, num_qo_heads, head_dim]
 *   k_cache  bf16 [num_pages, page_size, num_kv_heads, head_dim]   (NHD)
 *   v_cache  bf16 [num_pages, page_size, num_kv_heads, head_dim]
 *   o        bf16 [total_q, num_qo_heads, head_dim]
 *   lse      fp32 [total_q, num_qo_heads]
 *   MLA: q_nope bf16 [total_q, H, 512], q_pe bf16 [total_q, H, 64],
 *        ckv_cache bf16 [num_pages, page_size, 512],
 *        kpe_cache bf16 [num_pages, page_size, 64], o bf16 [total_q, H, 512].
 *   Device pointers must be 16-byte aligned. Slots past kv_last_page_len in a
 *   last page may hold any finite values; they are read but masked.
 *
 * Supported: bf16 (and FP8 E4M3 K/V pools for decode, pkv_run_fp8_kv);
 * sm_scale > 0; head_dim 64 or 128 (GQA), 512 + 64 (MLA); page_size a
 * power of two in [1, 256]; num_qo_heads % num_kv_heads == 0 with group size
 * <= 128 (<= 16 on the decode path). Anything else returns PKV_EUNSUPPORTED.
 *
 * Ownership and errors
 *   - The caller owns every device buffer and the workspace. A plan owns only
 *     host memory (including a pinned staging copy of its schedule).
 *   - No call throws; each returns a pkv_status. pkv_last_error() gives a
 *     thread-local message for the last failure on the calling thread.
 *   - pkv_run / pkv_run_mla never allocate and never synchronise: they only
 *     launch kernels on the given stream. Device-side waits are bounded: a wait
 *     that times out sets an error code in the workspace that
 *     pkv_device_status() reports (the outputs of that launch are then invalid).
 *   - Streams are passed as void* (a cudaStream_t; NULL = legacy default stream).
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pkv_status {
  PKV_OK = 0,
  PKV_EINVAL = 1,        /* malformed arguments (indptr not monotone, bad last_page_len, NULL, ...) */
  PKV_EUNSUPPORTED = 2,  /* well-formed but outside the supported shapes */
  PKV_ENOSPACE = 3,      /* workspace smaller than pkv_plan_workspace_bytes() */
  PKV_ECUDA = 4,         /* a CUDA runtime call failed (message in pkv_last_error) */
  PKV_EDEVICE = 5        /* a kernel reported an error through the device status word */
} pkv_status;

typedef struct pkv_plan pkv_plan; /* opaque; created by pkv_plan_create, freed by pkv_plan_destroy */

/* Scheduling knobs. Zero-initialise for the defaults. */
typedef struct pkv_plan_options {
  int32_t num_sms;          /* SMs to schedule for; 0 = query the current device */
  int32_t disable_split_kv; /* 1 = never split a request's KV across CTAs */
  int32_t kv_chunk;         /* >0: force this KV chunk length (tokens) when splitting; 0 = auto */
  int32_t kv_layout;        /* GQA/MHA page layout (FlashInfer 0.7.4 documentation, "KV-Cache Layout in
                               FlashInfer", "Layout: NHD/HND"): 0 = NHD, a page is [page_size, Hk, D];
                               1 = HND, a page is [Hk, page_size, D]. MLA pools have no head axis: ignored. */
  int32_t kv_fp8;           /* 1 = the plan is for pkv_run_fp8_kv. A decode plan's split-KV chunk is then sized
                               for the FP8 kernel's occupancy (results do not depend on it; either run accepts
                               either decode plan). A prefill plan reserves workspace for a bf16 copy of the
                               batch's pages, which pkv_run_fp8_kv needs (about 4 bytes per page element more).
                               Ignored by MLA plans. */
  int32_t reserved[3];
} pkv_plan_options;

/* Plan a batch: builds the CTA work list on the host.
 * Inputs (HOST int32 arrays): qo_indptr[batch+1], kv_indptr[batch+1] (pages),
 * kv_last_page_len[batch]. kv_indices is the DEVICE array of physical page ids
 * [kv_indptr[batch]]; the plan keeps the pointer (borrowed, not copied) and the
 * kernels read it at run time. head_dim is the QK and V width. For MLA use
 * pkv_plan_create_mla. opts may be NULL.
 * Returns PKV_EINVAL for malformed page tables, PKV_EUNSUPPORTED for shapes
 * outside the supported set. On success *out owns the plan. */
PKV_API pkv_status pkv_plan_create(const int32_t* qo_indptr, const int32_t* kv_indptr, const int32_t* kv_indices,
                           const int32_t* kv_last_page_len, int32_t batch, int32_t num_qo_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t page_size, int32_t causal,
                           float sm_scale, const pkv_plan_options* opts, pkv_plan** out);

/* Plan an absorbed-MLA batch: num_heads query heads share one latent KV
 * (ckv of width head_dim_ckv, rope key kpe of width head_dim_kpe). A batch
 * whose requests all have qo_len <= 1 and num_heads <= 16 is planned as MLA
 * decode (FlashInfer 0.2 release, "Fused MLA decode kernel": one CTA streams a
 * request's latent rows once for all its heads, split-KV + merge); any other
 * batch runs the tensor-core MLA prefill kernel. */
PKV_API pkv_status pkv_plan_create_mla(const int32_t* qo_indptr, const int32_t* kv_indptr, const int32_t* kv_indices,
                               const int32_t* kv_last_page_len, int32_t batch, int32_t num_heads,
                               int32_t head_dim_ckv, int32_t head_dim_kpe, int32_t page_size, int32_t causal,
                               float sm_scale, const pkv_plan_options* opts, pkv_plan** out);

/* Device workspace the plan needs (bytes, 256-byte aligned start). */
PKV_API size_t pkv_plan_workspace_bytes(const pkv_plan* plan);

/* Copy the schedule into `workspace` (DEVICE, >= pkv_plan_workspace_bytes) with
 * one asynchronous host-to-device copy on `stream` from the plan's pinned
 * staging buffer, and bind the plan to it. Call once before pkv_run; the
 * workspace must stay alive and untouched while the plan is used. */
PKV_API pkv_status pkv_plan_upload(pkv_plan* plan, void* workspace, size_t workspace_bytes, void* stream);

/* Run GQA / MHA attention (prefill or decode, chosen by the plan) on `stream`.
 * q, k_cache, v_cache: DEVICE bf16 as laid out above; num_pages = pool size
 * (page ids in kv_indices must be < num_pages; they are not checked on the
 * device). o: DEVICE bf16, lse: DEVICE fp32 (may be NULL to skip it).
 * Threading: any thread, any device (the kernels' shared-memory limits are
 * raised once per device, on its first launch). */
PKV_API pkv_status pkv_run(const pkv_plan* plan, const void* q, const void* k_cache, const void* v_cache,
                   int32_t num_pages, void* o, float* lse, void* stream);

/* Run absorbed-MLA attention on `stream` (plan from pkv_plan_create_mla). */
PKV_API pkv_status pkv_run_mla(const pkv_plan* plan, const void* q_nope, const void* q_pe, const void* ckv_cache,
                       const void* kpe_cache, int32_t num_pages, void* o, float* lse, void* stream);

/* Paged attention over a per-head-scale quantised KV cache ("[Roadmap]
 * FlashInfer v0.2 to v0.3", milestone "Per Head Scale Quantized KV-Cache").
 * The pools hold FP8 E4M3 codes (OCP 8-bit floating point: 1 sign bit, 4
 * exponent bits with bias 7, 3 mantissa bits, exponent field 0 subnormal,
 * S.1111.111 NaN), one byte per element, NHD pages:
 *   k_codes, v_codes  uint8 [num_pages, page_size, num_kv_heads, head_dim]  DEVICE
 *   k_scale, v_scale  fp32  [num_kv_heads]  DEVICE, or NULL for 1.0
 * The cache's value is decode(code) * scale[kv head], and the result is
 * pkv_run's attention over those values: q, o, lse as there. The plan is a
 * pkv_plan_create plan with the NHD layout and head_dim 64 or 128 (anything
 * else returns PKV_EUNSUPPORTED), either
 *   - a decode plan (every qo_len <= 1, group <= 16): one kernel reads the
 *     codes directly. On the device each CTA scales its Q rows by a power of
 *     two that brings their largest |q| to [2^13, 2^14) (undone exactly in the
 *     score scale) and rounds them to f16, so any finite bf16 q is accepted; P
 *     is rounded to f16, every code converts exactly to f16, and O and the LSE
 *     accumulate in fp32; or
 *   - a prefill plan made with pkv_plan_options.kv_fp8 = 1 (else
 *     PKV_EUNSUPPORTED): a first kernel writes the batch's pages as bf16 (every
 *     E4M3 value is exact in bf16; slots past a request's last key as zeros)
 *     into the plan's workspace, and the tensor-core prefill of pkv_run runs
 *     on that copy with K's scale applied to the scores and V's to the output;
 *     Q and P are bf16 as in pkv_run. The scales must then be positive.
 * NaN codes in a request's keys propagate. Pointers 16-byte aligned; num_pages
 * as in pkv_run. Never allocates, never synchronises; the split-KV merge runs
 * on the same stream. */
PKV_API pkv_status pkv_run_fp8_kv(const pkv_plan* plan, const void* q, const void* k_codes, const void* v_codes,
                                  const float* k_scale, const float* v_scale, int32_t num_pages, void* o,
                                  float* lse, void* stream);

/* Merge two attention states over disjoint key sets (all DEVICE fp32):
 * o_a, o_b, o_out [rows, dim]; lse_a, lse_b, lse_out [rows] (base 2).
 * lse_out = log2(2^lse_a + 2^lse_b), o_out = 2^(lse_a-lse_out) o_a + 2^(lse_b-lse_out) o_b.
 * o_out / lse_out may alias o_a / lse_a. dim <= 1024. */
PKV_API pkv_status pkv_merge_state(const float* o_a, const float* lse_a, const float* o_b, const float* lse_b,
                           float* o_out, float* lse_out, int32_t rows, int32_t dim, void* stream);

/* The same merge on bf16 outputs, as two attention runs produce them (FlashInfer
 * 0.7.4 documentation, flashinfer.cascade: "Merge Attention States" and
 * "Cascade Attention": a batch sharing a KV prefix attends to the prefix once
 * and to each request's own pages once, and the two states are merged).
 * o_a, o_b, o_out: DEVICE bf16 [rows, dim]; lse_*: DEVICE fp32 [rows], base 2.
 * Arithmetic in fp32; o_out / lse_out may alias o_a / lse_a. dim <= 1024. */
PKV_API pkv_status pkv_merge_state_bf16(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                                        void* o_out, float* lse_out, int32_t rows, int32_t dim, void* stream);

/* Merge `num` states (DEVICE fp32 o_parts [num, rows, dim], lse_parts [num, rows])
 * into bf16 o_out [rows, dim] and fp32 lse_out [rows]. dim <= 1024. */
PKV_API pkv_status pkv_merge_states(const float* o_parts, const float* lse_parts, int32_t num, int32_t rows,
                            int32_t dim, void* o_out, float* lse_out, void* stream);

/* Append new K/V rows to the paged cache (FlashInfer 0.2 release, "KV-Cache
 * append optimization": parallel over the new elements, not over requests;
 * positions as in the documentation's get_batch_indices_positions).
 * The page table (kv_indptr [batch+1], kv_indices, kv_last_page_len [batch];
 * all DEVICE int32) is the table AFTER the append: request b's new rows,
 * k_new / v_new rows append_indptr[b] .. append_indptr[b+1] - 1 (DEVICE int32
 * [batch+1], nnz = append_indptr[batch] rows in total), are written to its last
 * positions kv_len - n .. kv_len - 1 (n = its row count), i.e. page
 * kv_indices[kv_indptr[b] + pos / page_size], slot pos % page_size.
 * k_new [nnz, num_kv_heads, head_dim], v_new [nnz, num_kv_heads, head_dim_v]:
 * DEVICE bf16 (any 2-byte type: bytes are copied unchanged). k_cache
 * [num_pages, page_size, num_kv_heads, head_dim] (kv_layout 0, NHD) or
 * [num_pages, num_kv_heads, page_size, head_dim] (kv_layout 1, HND), v_cache
 * likewise with head_dim_v: DEVICE, updated in place; every other slot is left
 * untouched.
 * MLA caches fit the same call with num_kv_heads 1: k = ckv (512), v = kpe (64).
 * Head dims must be multiples of 8 and pointers 16-byte aligned.
 * A row whose position falls outside its request, or whose page id is not in
 * [0, num_pages), is skipped and, if `status` (DEVICE int32, may be NULL) is
 * given, sets *status = 1. Launch only: no allocation, no synchronisation. */
PKV_API pkv_status pkv_append_kv(const void* k_new, const void* v_new, const int32_t* append_indptr, int64_t nnz,
                                 const int32_t* kv_indptr, const int32_t* kv_indices,
                                 const int32_t* kv_last_page_len, int32_t batch, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t head_dim_v, int32_t page_size, int32_t num_pages,
                                 int32_t kv_layout, void* k_cache, void* v_cache, int32_t* status, void* stream);

/* Paged decode (one query token per request) for callers that cannot allocate
 * device memory: code under an allocator that forbids new device allocations
 * (a fixed pool, an embedded host that only registers buffers at start-up) or
 * a serving thread that must not enter the allocator. It needs no plan and no
 * workspace: the page table is read on the device, nothing is uploaded, and
 * split-KV partial states live in one fixed 16 MiB device array inside the
 * library (allocated when the library is loaded, held by every GPU that loads
 * it until exit). The pages this library follows have no counterpart of this
 * call; it computes the same result as pkv_run on a decode plan.
 *   q [batch, num_qo_heads, head_dim], k_cache / v_cache as for pkv_run,
 *   kv_indptr [batch+1], kv_indices, kv_last_page_len [batch]: all DEVICE int32.
 *   max_kv_len: an upper bound on the requests' kv_len, used to size the split
 *   (a larger kv_len is still computed exactly, only more slowly).
 *   o [batch, num_qo_heads, head_dim] bf16, lse [batch, num_qo_heads] fp32 (or NULL).
 * Supports num_qo_heads / num_kv_heads <= 16, head_dim 64 or 128, batch and
 * num_kv_heads up to 65535; q, k_cache, v_cache and o 16-byte aligned, the
 * index arrays and lse 4-byte aligned (else PKV_EINVAL, nothing launched).
 * The split gives every SM about four CTAs with chunks of at least 256 keys;
 * a request whose KV fits one chunk writes O / LSE directly, others go through
 * the scratch and one merge launch. That rule needs at most about 70 KB of
 * scratch per SM of the device (about 10 MB on a 148-SM B200), so the
 * PKV_ENOSPACE refusal (returned without launching anything when a split would
 * need more than the 16 MiB) can only occur on a GPU with more than 240 SMs.
 * The first call on each device looks up the
 * scratch address (cudaGetSymbolAddress) and should come before any stream
 * capture. All calls share the scratch: calls whose kernels overlap on the GPU
 * (other streams, unordered threads) race on it and must be serialised. */
PKV_API pkv_status pkv_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* kv_indptr, const int32_t* kv_indices,
                                      const int32_t* kv_last_page_len, int32_t batch, int32_t num_qo_heads,
                                      int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                                      int32_t max_kv_len, float sm_scale, void* o, float* lse, void* stream);

/* Self-test of the bounded device-side waits (no GPU fault involved): one CTA
 * waits on an mbarrier that nothing arrives on, through the same bounded wait
 * every kernel uses. Expected on return (after about 2 s): *status (DEVICE
 * int32, zero on entry) = 1, the wait-timeout code; times[0] (DEVICE int64) =
 * nanoseconds the first wait took before giving up (about 2e9); times[1] = the
 * nanoseconds a second wait took once the CTA was aborting (a few hundred),
 * or -1 where a wait unexpectedly completed. The CUDA context stays usable. */
PKV_API pkv_status pkv_selftest_wait_timeout(int32_t* status, int64_t* times, void* stream);

/* Read the device status word of the plan's workspace (synchronises `stream`).
 * PKV_OK if no kernel reported an error; PKV_EDEVICE otherwise (and the code is
 * stored in *code if code != NULL). */
PKV_API pkv_status pkv_device_status(const pkv_plan* plan, void* stream, int32_t* code);

/* Introspection (host only, no device access):
 *   key 0 kernel kind (0 prefill, 1 decode, 2 MLA, 3 MLA decode), 1 work units, 2 merge tasks,
 *   3 partial slots, 4 rows per partial slot, 5 SMs planned for, 6 KV chunk,
 *   7 CTAs of the main launch (prefill: persistent CTAs, each running a fixed
 *   list of work units; decode / MLA: one CTA per work unit). */
PKV_API int64_t pkv_plan_info(const pkv_plan* plan, int32_t key);

/* Copy the work list (8 int32 per unit: req, kv_head, row0, rows, kv_lo, kv_hi,
 * partial slot or -1, 0) into `out` (HOST, capacity in units). Returns units copied. */
PKV_API int32_t pkv_plan_work_units(const pkv_plan* plan, int32_t* out, int32_t capacity);

/* Copy the merge list (8 int32 per task: req, kv_head, row0, rows, slot0, num, 0, 0). */
PKV_API int32_t pkv_plan_merge_tasks(const pkv_plan* plan, int32_t* out, int32_t capacity);

/* Copy the persistent-CTA schedule of a prefill plan: num_ctas + 1 offsets
 * into the work list (CTA b runs units [out[b], out[b + 1]) in order) into
 * `out` (HOST, capacity in int32). Returns the entries copied; 0 for decode and
 * MLA plans, whose CTAs each run one unit. */
PKV_API int32_t pkv_plan_cta_units(const pkv_plan* plan, int32_t* out, int32_t capacity);

PKV_API void pkv_plan_destroy(pkv_plan* plan);

/* Message for the last failure on this thread ("" if none). */
PKV_API const char* pkv_last_error(void);

/* Library version string. */
PKV_API const char* pkv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
