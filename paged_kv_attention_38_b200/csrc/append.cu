// Appending new K/V rows to the paged cache.
//
// FlashInfer 0.2 release, "KV-Cache append optimization": the append is
// parallelised over the new elements rather than over requests, so a batch
// with a few long appends (prefill) and many single-token ones (decode) keeps
// every SM busy. The page table passed in is the one after the append
// (documentation, "Page Table Layout"; get_batch_indices_positions): request
// b's n new rows take its last n positions kv_len - n .. kv_len - 1.
//
// One thread moves one 16-byte piece of one (new row, kv head) of K and the
// same piece of V: consecutive threads cover consecutive bytes of a row, so
// both the reads of the new rows and the writes into a page slot are
// coalesced. The request of a new row comes from a binary search over
// append_indptr (a few steps, the array stays in L1).
#include <cuda_runtime.h>

#include <cstdint>
#include <string>

#include "pkv.h"

namespace pkv {
void set_last_error(const std::string& msg);

namespace {

constexpr int kThreads = 256;

struct AppendArgs {
  const uint4* k_new;  // [nnz, Hk, Dk] bf16, as 16-byte pieces
  const uint4* v_new;  // [nnz, Hk, Dv]
  const int32_t* append_indptr;
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* kv_last_page_len;
  uint4* k_cache;      // [num_pages, P, Hk, Dk] (NHD) or [num_pages, Hk, P, Dk] (HND)
  uint4* v_cache;      // likewise with Dv
  int32_t* status;     // optional: set to 1 when a row had no valid slot
  int32_t batch, num_kv_heads, chunks_k, chunks_v, page_size, num_pages;
  int32_t hnd;         // pages laid out [kv head][slot][D] instead of [slot][kv head][D]
  int64_t nnz;
};

__global__ void __launch_bounds__(kThreads) append_kernel(const AppendArgs a) {
  const int chunks = a.chunks_k > a.chunks_v ? a.chunks_k : a.chunks_v;
  const int64_t per_row = (int64_t)a.num_kv_heads * chunks;
  const int64_t total = a.nnz * per_row;
  for (int64_t e = (int64_t)blockIdx.x * kThreads + threadIdx.x; e < total; e += (int64_t)gridDim.x * kThreads) {
    const int64_t t = e / per_row;  // new row
    const int rem = (int)(e - t * per_row);
    const int h = rem / chunks, c = rem % chunks;
    // request b with append_indptr[b] <= t < append_indptr[b + 1]
    int lo = 0, hi = a.batch;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(a.append_indptr + mid) <= t) lo = mid;
      else hi = mid;
    }
    const int b = lo;
    const int a0 = __ldg(a.append_indptr + b), n = __ldg(a.append_indptr + b + 1) - a0;
    const int p0 = __ldg(a.kv_indptr + b), np = __ldg(a.kv_indptr + b + 1) - p0;
    const int64_t kv_len = np > 0 ? (int64_t)(np - 1) * a.page_size + __ldg(a.kv_last_page_len + b) : 0;
    const int64_t pos = kv_len - n + (t - a0);
    if (pos < 0 || pos >= kv_len) {  // more new rows than the table holds: skip, report
      if (a.status) atomicExch(a.status, 1);
      continue;
    }
    const int page = __ldg(a.kv_indices + p0 + (int)(pos / a.page_size));
    if (page < 0 || page >= a.num_pages) {
      if (a.status) atomicExch(a.status, 1);
      continue;
    }
    const int64_t slot_row = a.hnd ? ((int64_t)page * a.num_kv_heads + h) * a.page_size + pos % a.page_size
                                   : ((int64_t)page * a.page_size + pos % a.page_size) * a.num_kv_heads + h;
    const int64_t new_row = t * a.num_kv_heads + h;
    if (c < a.chunks_k) a.k_cache[slot_row * a.chunks_k + c] = a.k_new[new_row * a.chunks_k + c];
    if (c < a.chunks_v) a.v_cache[slot_row * a.chunks_v + c] = a.v_new[new_row * a.chunks_v + c];
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

}  // namespace
}  // namespace pkv

extern "C" pkv_status pkv_append_kv(const void* k_new, const void* v_new, const int32_t* append_indptr, int64_t nnz,
                                    const int32_t* kv_indptr, const int32_t* kv_indices,
                                    const int32_t* kv_last_page_len, int32_t batch, int32_t num_kv_heads,
                                    int32_t head_dim, int32_t head_dim_v, int32_t page_size, int32_t num_pages,
                                    int32_t kv_layout, void* k_cache, void* v_cache, int32_t* status, void* stream) {
  using namespace pkv;
  if (batch < 0 || nnz < 0) {
    set_last_error("batch and nnz must be non-negative");
    return PKV_EINVAL;
  }
  if (batch == 0 || nnz == 0) return PKV_OK;
  if (num_kv_heads <= 0 || head_dim <= 0 || head_dim_v <= 0 || head_dim % 8 != 0 || head_dim_v % 8 != 0) {
    set_last_error("num_kv_heads > 0 and head dims that are positive multiples of 8 required");
    return PKV_EUNSUPPORTED;
  }
  if (kv_layout != 0 && kv_layout != 1) {
    set_last_error("kv_layout must be 0 (NHD) or 1 (HND)");
    return PKV_EINVAL;
  }
  if (page_size <= 0 || num_pages <= 0) {
    set_last_error("page_size and num_pages must be positive");
    return PKV_EINVAL;
  }
  if (!k_new || !v_new || !append_indptr || !kv_indptr || !kv_indices || !kv_last_page_len || !k_cache ||
      !v_cache) {
    set_last_error("NULL pointer");
    return PKV_EINVAL;
  }
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache)) {
    set_last_error("K/V pointers must be 16-byte aligned");
    return PKV_EINVAL;
  }
  AppendArgs a{};
  a.k_new = static_cast<const uint4*>(k_new);
  a.v_new = static_cast<const uint4*>(v_new);
  a.append_indptr = append_indptr;
  a.kv_indptr = kv_indptr;
  a.kv_indices = kv_indices;
  a.kv_last_page_len = kv_last_page_len;
  a.k_cache = static_cast<uint4*>(k_cache);
  a.v_cache = static_cast<uint4*>(v_cache);
  a.status = status;
  a.batch = batch;
  a.num_kv_heads = num_kv_heads;
  a.chunks_k = head_dim / 8;
  a.chunks_v = head_dim_v / 8;
  a.page_size = page_size;
  a.num_pages = num_pages;
  a.nnz = nnz;
  a.hnd = kv_layout;
  const int64_t total = nnz * num_kv_heads * (a.chunks_k > a.chunks_v ? a.chunks_k : a.chunks_v);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  const int64_t blocks = (total + kThreads - 1) / kThreads;
  const int grid = (int)(blocks < (int64_t)sms * 8 ? blocks : (int64_t)sms * 8);
  append_kernel<<<grid, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error(std::string("append: ") + cudaGetErrorString(e));
    return PKV_ECUDA;
  }
  return PKV_OK;
}
