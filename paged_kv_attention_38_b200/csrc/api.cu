// C ABI of libpkv.so (declared in include/pkv.h): plan objects, the one
// host-to-device copy of a schedule, and the launches behind pkv_run.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>

#include "pkv.h"
#include "pkv_internal.h"
#include "planner.h"

namespace pkv {
cudaError_t launch_prefill(const LaunchGeom&, const DeviceView&, const int32_t*, const void*, const void*,
                           const void*, int32_t, void*, float*, const float*, const float*, cudaStream_t);
cudaError_t launch_kv_fp8_expand(const LaunchGeom&, const DeviceView&, const int32_t*, int32_t, const void*,
                                 const void*, void*, void*, int32_t*, cudaStream_t);
cudaError_t launch_decode(const LaunchGeom&, const DeviceView&, const int32_t*, const void*, const void*,
                          const void*, void*, float*, cudaStream_t);
cudaError_t launch_mla(const LaunchGeom&, const DeviceView&, const int32_t*, const void*, const void*,
                       const void*, const void*, void*, float*, cudaStream_t);
cudaError_t launch_mla_decode(const LaunchGeom&, const DeviceView&, const int32_t*, const void*, const void*,
                              const void*, const void*, void*, float*, cudaStream_t);
cudaError_t launch_decode_fp8(const LaunchGeom&, const DeviceView&, const int32_t*, const void*, const void*,
                              const void*, const float*, const float*, void*, float*, cudaStream_t);
cudaError_t launch_merge_tasks(const LaunchGeom&, const DeviceView&, void*, float*, cudaStream_t);
cudaError_t launch_merge_state(const float*, const float*, const float*, const float*, float*, float*, int, int,
                               cudaStream_t);
cudaError_t launch_merge_states(const float*, const float*, int, int, int, void*, float*, cudaStream_t);
cudaError_t launch_merge_state_bf16(const void*, const float*, const void*, const float*, void*, float*, int, int,
                                    cudaStream_t);
}  // namespace pkv

using namespace pkv;

struct pkv_plan {
  Schedule sched;
  const int32_t* kv_indices = nullptr;  // device, borrowed
  // workspace layout (byte offsets)
  size_t off_status = 0, off_units = 0, off_merges = 0, off_reqs = 0, off_cta = 0, off_row0 = 0, off_lse = 0, off_o = 0,
         off_packed = 0, off_fp8_k = 0, off_fp8_v = 0, off_fp8_idx = 0, total = 0;
  bool kv_fp8 = false;          // planned for pkv_run_fp8_kv (kv_fp8 option)
  uint8_t* ws = nullptr;        // device workspace (set by pkv_plan_upload)
  int32_t page_entries = 0;     // kv_indptr[batch]: entries of the page table
  size_t staging_bytes = 0;
  void* staging = nullptr;  // host copy of [status | units | merges | reqs | cta_ptr]
  bool staging_pinned = false;
  DeviceView dv{};
  bool uploaded = false;
};

namespace {

thread_local std::string g_err;

pkv_status fail(pkv_status s, const std::string& msg) {
  g_err = msg;
  return s;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

int query_num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    return 148;
  }
  return n;
}

void layout_workspace(pkv_plan* p) {
  const Schedule& s = p->sched;
  size_t off = 0;
  p->off_status = off;
  off += 256;
  p->off_units = off;
  off = align256(off + s.units.size() * sizeof(WorkUnit));
  p->off_merges = off;
  off = align256(off + s.merges.size() * sizeof(MergeTask));
  p->off_reqs = off;
  off = align256(off + s.reqs.size() * sizeof(ReqInfo));
  p->off_cta = off;
  off = align256(off + s.cta_ptr.size() * sizeof(int32_t));
  p->off_row0 = off;
  off = align256(off + s.kv_row0.size() * sizeof(int32_t));
  p->staging_bytes = off;
  p->off_lse = off;
  off = align256(off + (size_t)s.num_slots * s.geom.part_rows * sizeof(float));
  p->off_o = off;
  off = align256(off + (size_t)s.num_slots * s.geom.part_rows * s.geom.head_dim_v * sizeof(float));
  p->off_packed = off;
  if (s.kind == kKindMla)  // the packed latent copy, ckv | kpe per key (at least one row for the tensor map)
    off = align256(off + (size_t)std::max(1, s.geom.packed_rows) * (s.geom.head_dim + s.geom.head_dim_pe) * 2);
  // prefill over an FP8 cache: bf16 copies of the batch's K and V pages
  // ([entries][page_size][Hk][D]) and their identity page table
  const size_t fp8_page_bytes =
      p->kv_fp8 && s.kind == kKindPrefill
          ? (size_t)s.geom.page_size * s.geom.num_kv_heads * s.geom.head_dim * 2 : 0;
  const size_t fp8_entries = fp8_page_bytes ? (size_t)std::max(1, p->page_entries) : 0;
  p->off_fp8_k = off;
  off = align256(off + fp8_entries * fp8_page_bytes);
  p->off_fp8_v = off;
  off = align256(off + fp8_entries * fp8_page_bytes);
  p->off_fp8_idx = off;
  off = align256(off + fp8_entries * sizeof(int32_t));
  p->total = off;
}

pkv_status create_common(const PlanInput& in, const int32_t* kv_indices, pkv_plan** out) {
  if (!out) return fail(PKV_EINVAL, "out is NULL");
  *out = nullptr;
  pkv_plan* p = new (std::nothrow) pkv_plan();
  if (!p) return fail(PKV_EINVAL, "out of host memory");
  std::string err;
  const int rc = build_schedule(in, &p->sched, &err);
  if (rc != 0) {
    delete p;
    return fail(rc == 1 ? PKV_EINVAL : PKV_EUNSUPPORTED, err);
  }
  p->kv_indices = kv_indices;
  p->kv_fp8 = in.kv_fp8 != 0;
  p->page_entries = in.batch > 0 ? in.kv_indptr[in.batch] : 0;
  layout_workspace(p);
  *out = p;
  return PKV_OK;
}

void fill_in(PlanInput& in, const int32_t* qo_indptr, const int32_t* kv_indptr, const int32_t* last, int32_t batch,
             int32_t page_size, int32_t causal, float sm_scale, const pkv_plan_options* opts) {
  in.qo_indptr = qo_indptr;
  in.kv_indptr = kv_indptr;
  in.kv_last_page_len = last;
  in.batch = batch;
  in.page_size = page_size;
  in.causal = causal;
  in.sm_scale = sm_scale;
  in.num_sms = (opts && opts->num_sms > 0) ? opts->num_sms : query_num_sms();
  in.disable_split_kv = opts ? opts->disable_split_kv : 0;
  in.kv_chunk = opts ? opts->kv_chunk : 0;
  in.kv_layout = opts ? opts->kv_layout : 0;
  in.kv_fp8 = opts ? opts->kv_fp8 : 0;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace

namespace pkv {
// Lets other translation units of the library report through pkv_last_error().
void set_last_error(const std::string& msg) { g_err = msg; }
}  // namespace pkv

extern "C" {

pkv_status pkv_plan_create(const int32_t* qo_indptr, const int32_t* kv_indptr, const int32_t* kv_indices,
                           const int32_t* kv_last_page_len, int32_t batch, int32_t num_qo_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t page_size, int32_t causal,
                           float sm_scale, const pkv_plan_options* opts, pkv_plan** out) {
  PlanInput in{};
  fill_in(in, qo_indptr, kv_indptr, kv_last_page_len, batch, page_size, causal, sm_scale, opts);
  in.num_qo_heads = num_qo_heads;
  in.num_kv_heads = num_kv_heads;
  in.head_dim = head_dim;
  in.head_dim_v = head_dim;
  in.head_dim_pe = 0;
  return create_common(in, kv_indices, out);
}

pkv_status pkv_plan_create_mla(const int32_t* qo_indptr, const int32_t* kv_indptr, const int32_t* kv_indices,
                               const int32_t* kv_last_page_len, int32_t batch, int32_t num_heads,
                               int32_t head_dim_ckv, int32_t head_dim_kpe, int32_t page_size, int32_t causal,
                               float sm_scale, const pkv_plan_options* opts, pkv_plan** out) {
  PlanInput in{};
  fill_in(in, qo_indptr, kv_indptr, kv_last_page_len, batch, page_size, causal, sm_scale, opts);
  in.num_qo_heads = num_heads;
  in.num_kv_heads = 1;
  in.head_dim = head_dim_ckv;
  in.head_dim_v = head_dim_ckv;
  in.head_dim_pe = head_dim_kpe;
  if (head_dim_kpe <= 0) return fail(PKV_EUNSUPPORTED, "MLA needs head_dim_kpe > 0");
  return create_common(in, kv_indices, out);
}

size_t pkv_plan_workspace_bytes(const pkv_plan* plan) { return plan ? plan->total : 0; }

pkv_status pkv_plan_upload(pkv_plan* p, void* workspace, size_t bytes, void* stream) {
  if (!p) return fail(PKV_EINVAL, "plan is NULL");
  if (!workspace) return fail(PKV_EINVAL, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return fail(PKV_EINVAL, "workspace must be 256-byte aligned");
  if (bytes < p->total) return fail(PKV_ENOSPACE, "workspace smaller than pkv_plan_workspace_bytes()");
  if (!p->staging) {
    if (cudaMallocHost(&p->staging, p->staging_bytes) == cudaSuccess) {
      p->staging_pinned = true;
    } else {
      cudaGetLastError();
      p->staging = std::malloc(p->staging_bytes);
      if (!p->staging) return fail(PKV_EINVAL, "out of host memory");
    }
    uint8_t* h = static_cast<uint8_t*>(p->staging);
    std::memset(h, 0, p->staging_bytes);
    const Schedule& s = p->sched;
    if (!s.units.empty()) std::memcpy(h + p->off_units, s.units.data(), s.units.size() * sizeof(WorkUnit));
    if (!s.merges.empty()) std::memcpy(h + p->off_merges, s.merges.data(), s.merges.size() * sizeof(MergeTask));
    if (!s.reqs.empty()) std::memcpy(h + p->off_reqs, s.reqs.data(), s.reqs.size() * sizeof(ReqInfo));
    if (!s.cta_ptr.empty()) std::memcpy(h + p->off_cta, s.cta_ptr.data(), s.cta_ptr.size() * sizeof(int32_t));
    if (!s.kv_row0.empty()) std::memcpy(h + p->off_row0, s.kv_row0.data(), s.kv_row0.size() * sizeof(int32_t));
  }
  uint8_t* d = static_cast<uint8_t*>(workspace);
  cudaError_t e = cudaMemcpyAsync(d, p->staging, p->staging_bytes, cudaMemcpyHostToDevice,
                                  static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("upload: ") + cudaGetErrorString(e));
  p->dv.units = reinterpret_cast<const WorkUnit*>(d + p->off_units);
  p->dv.merges = reinterpret_cast<const MergeTask*>(d + p->off_merges);
  p->dv.reqs = reinterpret_cast<const ReqInfo*>(d + p->off_reqs);
  p->dv.part_lse = reinterpret_cast<float*>(d + p->off_lse);
  p->dv.part_o = reinterpret_cast<float*>(d + p->off_o);
  p->dv.status = reinterpret_cast<int*>(d + p->off_status);
  p->dv.cta_ptr = reinterpret_cast<const int32_t*>(d + p->off_cta);
  p->dv.kv_row0 = reinterpret_cast<const int32_t*>(d + p->off_row0);
  p->dv.packed = d + p->off_packed;
  p->ws = d;
  p->uploaded = true;
  return PKV_OK;
}

pkv_status pkv_run(const pkv_plan* p, const void* q, const void* k_cache, const void* v_cache, int32_t num_pages,
                   void* o, float* lse, void* stream) {
  if (!p) return fail(PKV_EINVAL, "plan is NULL");
  if (!p->uploaded) return fail(PKV_EINVAL, "plan not uploaded (call pkv_plan_upload)");
  const Schedule& s = p->sched;
  if (s.kind == kKindMla || s.kind == kKindMlaDecode) return fail(PKV_EINVAL, "MLA plan: use pkv_run_mla");
  if (s.units.empty()) return PKV_OK;
  if (!q || !k_cache || !v_cache || !o || !p->kv_indices) return fail(PKV_EINVAL, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(o))
    return fail(PKV_EINVAL, "tensor pointers must be 16-byte aligned");
  if (num_pages <= 0) return fail(PKV_EINVAL, "num_pages must be positive");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = s.kind == kKindDecode
                      ? launch_decode(s.geom, p->dv, p->kv_indices, q, k_cache, v_cache, o, lse, st)
                      : launch_prefill(s.geom, p->dv, p->kv_indices, q, k_cache, v_cache, num_pages, o, lse,
                                       nullptr, nullptr, st);
  if (e == cudaSuccess) e = launch_merge_tasks(s.geom, p->dv, o, lse, st);
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("launch: ") + cudaGetErrorString(e));
  return PKV_OK;
}

pkv_status pkv_run_mla(const pkv_plan* p, const void* q_nope, const void* q_pe, const void* ckv_cache,
                       const void* kpe_cache, int32_t num_pages, void* o, float* lse, void* stream) {
  if (!p) return fail(PKV_EINVAL, "plan is NULL");
  if (!p->uploaded) return fail(PKV_EINVAL, "plan not uploaded (call pkv_plan_upload)");
  const Schedule& s = p->sched;
  if (s.kind != kKindMla && s.kind != kKindMlaDecode) return fail(PKV_EINVAL, "not an MLA plan: use pkv_run");
  if (s.units.empty()) return PKV_OK;
  if (!q_nope || !q_pe || !ckv_cache || !kpe_cache || !o || !p->kv_indices)
    return fail(PKV_EINVAL, "NULL tensor pointer");
  if (!aligned16(q_nope) || !aligned16(q_pe) || !aligned16(ckv_cache) || !aligned16(kpe_cache) || !aligned16(o))
    return fail(PKV_EINVAL, "tensor pointers must be 16-byte aligned");
  if (num_pages <= 0) return fail(PKV_EINVAL, "num_pages must be positive");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = s.kind == kKindMlaDecode
                      ? launch_mla_decode(s.geom, p->dv, p->kv_indices, q_nope, q_pe, ckv_cache, kpe_cache, o, lse, st)
                      : launch_mla(s.geom, p->dv, p->kv_indices, q_nope, q_pe, ckv_cache, kpe_cache, o, lse, st);
  if (e == cudaSuccess) e = launch_merge_tasks(s.geom, p->dv, o, lse, st);
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("launch: ") + cudaGetErrorString(e));
  return PKV_OK;
}

pkv_status pkv_run_fp8_kv(const pkv_plan* p, const void* q, const void* k_codes, const void* v_codes,
                          const float* k_scale, const float* v_scale, int32_t num_pages, void* o, float* lse,
                          void* stream) {
  if (!p) return fail(PKV_EINVAL, "plan is NULL");
  const Schedule& s = p->sched;
  if (s.kind != kKindDecode && s.kind != kKindPrefill) return fail(PKV_EINVAL, "MLA plan: FP8 KV cache is GQA/MHA only");
  if (s.kind == kKindPrefill && !p->kv_fp8)
    return fail(PKV_EUNSUPPORTED, "FP8 KV cache with a prefill plan: create the plan with pkv_plan_options.kv_fp8 = 1 "
                                  "(it reserves the workspace for the bf16 copy of the pages)");
  if (s.geom.kv_layout != 0) return fail(PKV_EUNSUPPORTED, "FP8 KV cache: NHD pages only");
  if (s.geom.head_dim != 64 && s.geom.head_dim != 128)
    return fail(PKV_EUNSUPPORTED, "FP8 KV cache: head_dim 64 or 128");
  if (!p->uploaded) return fail(PKV_EINVAL, "plan not uploaded (call pkv_plan_upload)");
  if (s.units.empty()) return PKV_OK;
  if (!q || !k_codes || !v_codes || !o || !p->kv_indices) return fail(PKV_EINVAL, "NULL tensor pointer");
  if (!aligned16(q) || !aligned16(k_codes) || !aligned16(v_codes) || !aligned16(o))
    return fail(PKV_EINVAL, "tensor pointers must be 16-byte aligned");
  if (num_pages <= 0) return fail(PKV_EINVAL, "num_pages must be positive");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaSuccess;
  if (s.kind == kKindDecode) {
    e = launch_decode_fp8(s.geom, p->dv, p->kv_indices, q, k_codes, v_codes, k_scale, v_scale, o, lse, st);
  } else {
    // the batch's pages as bf16 in the workspace, then the tensor-core prefill on
    // that copy through an identity page table, the scales applied per kv head
    void* kc = p->ws + p->off_fp8_k;
    void* vc = p->ws + p->off_fp8_v;
    int32_t* idx = reinterpret_cast<int32_t*>(p->ws + p->off_fp8_idx);
    e = launch_kv_fp8_expand(s.geom, p->dv, p->kv_indices, p->page_entries, k_codes, v_codes, kc, vc, idx, st);
    if (e == cudaSuccess)
      e = launch_prefill(s.geom, p->dv, idx, q, kc, vc, std::max(1, p->page_entries), o, lse, k_scale, v_scale, st);
  }
  if (e == cudaSuccess) e = launch_merge_tasks(s.geom, p->dv, o, lse, st);
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("launch: ") + cudaGetErrorString(e));
  return PKV_OK;
}

pkv_status pkv_merge_state(const float* o_a, const float* lse_a, const float* o_b, const float* lse_b,
                           float* o_out, float* lse_out, int32_t rows, int32_t dim, void* stream) {
  if (rows < 0 || dim <= 0 || dim > 1024) return fail(PKV_EINVAL, "rows >= 0 and 0 < dim <= 1024 required");
  if (rows > 0 && (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out)) return fail(PKV_EINVAL, "NULL pointer");
  cudaError_t e = launch_merge_state(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, dim,
                                     static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("merge_state: ") + cudaGetErrorString(e));
  return PKV_OK;
}

pkv_status pkv_merge_state_bf16(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                                void* o_out, float* lse_out, int32_t rows, int32_t dim, void* stream) {
  if (rows < 0 || dim <= 0 || dim > 1024) return fail(PKV_EINVAL, "rows >= 0 and 0 < dim <= 1024 required");
  if (rows > 0 && (!o_a || !lse_a || !o_b || !lse_b || !o_out || !lse_out)) return fail(PKV_EINVAL, "NULL pointer");
  cudaError_t e = launch_merge_state_bf16(o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, dim,
                                          static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("merge_state_bf16: ") + cudaGetErrorString(e));
  return PKV_OK;
}

pkv_status pkv_merge_states(const float* o_parts, const float* lse_parts, int32_t num, int32_t rows, int32_t dim,
                            void* o_out, float* lse_out, void* stream) {
  if (num <= 0 || rows < 0 || dim <= 0 || dim > 1024) return fail(PKV_EINVAL, "num > 0, rows >= 0, 0 < dim <= 1024");
  if (rows > 0 && (!o_parts || !lse_parts || !o_out || !lse_out)) return fail(PKV_EINVAL, "NULL pointer");
  cudaError_t e = launch_merge_states(o_parts, lse_parts, num, rows, dim, o_out, lse_out,
                                      static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("merge_states: ") + cudaGetErrorString(e));
  return PKV_OK;
}

pkv_status pkv_device_status(const pkv_plan* p, void* stream, int32_t* code) {
  if (!p || !p->uploaded) return fail(PKV_EINVAL, "plan not uploaded");
  int32_t h = 0;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&h, p->dv.status, sizeof(int32_t), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return fail(PKV_ECUDA, std::string("status: ") + cudaGetErrorString(e));
  if (code) *code = h;
  if (h != 0) return fail(PKV_EDEVICE, "a kernel reported a device-side wait timeout");
  return PKV_OK;
}

int64_t pkv_plan_info(const pkv_plan* p, int32_t key) {
  if (!p) return -1;
  const Schedule& s = p->sched;
  switch (key) {
    case 0: return s.kind;
    case 1: return (int64_t)s.units.size();
    case 2: return (int64_t)s.merges.size();
    case 3: return s.num_slots;
    case 4: return s.geom.part_rows;
    case 5: return s.num_sms;
    case 6: return s.kv_chunk;
    case 7: return s.geom.num_ctas;
    default: return -1;
  }
}

int32_t pkv_plan_work_units(const pkv_plan* p, int32_t* out, int32_t capacity) {
  if (!p || !out || capacity <= 0) return 0;
  const int32_t n = (int32_t)std::min<size_t>(p->sched.units.size(), (size_t)capacity);
  std::memcpy(out, p->sched.units.data(), (size_t)n * sizeof(WorkUnit));
  return n;
}

int32_t pkv_plan_merge_tasks(const pkv_plan* p, int32_t* out, int32_t capacity) {
  if (!p || !out || capacity <= 0) return 0;
  const int32_t n = (int32_t)std::min<size_t>(p->sched.merges.size(), (size_t)capacity);
  std::memcpy(out, p->sched.merges.data(), (size_t)n * sizeof(MergeTask));
  return n;
}

int32_t pkv_plan_cta_units(const pkv_plan* p, int32_t* out, int32_t capacity) {
  if (!p || !out || capacity <= 0) return 0;
  const int32_t n = (int32_t)std::min<size_t>(p->sched.cta_ptr.size(), (size_t)capacity);
  if (n > 0) std::memcpy(out, p->sched.cta_ptr.data(), (size_t)n * sizeof(int32_t));
  return n;
}

void pkv_plan_destroy(pkv_plan* p) {
  if (!p) return;
  if (p->staging) {
    if (p->staging_pinned) cudaFreeHost(p->staging);  // waits for the copy that reads it
    else std::free(p->staging);
  }
  delete p;
}

const char* pkv_last_error(void) { return g_err.c_str(); }

const char* pkv_version(void) { return "pkv 0.1.0 (sm_100a)"; }

}  // extern "C"
