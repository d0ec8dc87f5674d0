// Paged decode for callers that cannot allocate device memory.
//
// pkv_run needs a device workspace (the uploaded work list, split-KV partial
// states and a status word) that the caller allocates. Some callers cannot do
// that: code running under an allocator that forbids new device allocations
// (a fixed memory pool, an embedded or real-time host that only pre-registers
// buffers at start-up), or a host thread that must not take the allocator's
// locks while it serves a request. pkv_decode_noalloc serves them: it takes the
// page table already on the device, builds no schedule on the host, uploads
// nothing and keeps its split-KV partial states in one file-scope device array
// (kNoAllocScratchBytes, 16 MiB, held by every GPU that loads the library until
// the process exits). It calls no cudaMalloc / cudaFree and no allocating
// library routine.
//
// The device address of that array is looked up once per device, on the first
// call made with that device current, with cudaGetSymbolAddress (host code must
// never pass the array's name itself to a kernel: on the host it is only a
// stand-in symbol, not a device address). That first call should therefore be
// made before any stream capture begins on the calling thread.
//
// Every call uses the same array, and the array keeps whatever the last call
// wrote: each call writes every partial slot it later reads, so nothing needs
// clearing, but two calls whose kernels overlap on the GPU (different streams,
// or one stream shared by several host threads without ordering) race on it.
//
// The attention itself is the planned decode's body (decode::attend in
// decode_core.cuh); only the CTA's job differs: it takes its (request, kv
// head, KV chunk) from blockIdx and reads the request's length from the device
// page table, instead of from an uploaded work list.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <string>

#include "decode_core.cuh"
#include "launch_util.h"
#include "pkv.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

// Largest scratch any call may use; calls that would need more are rejected.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void set_last_error(const std::string& msg);  // api.cu

namespace {

constexpr int kRowsMax = 16;       // query heads per kv head handled by one CTA
constexpr int kMaxDevices = 64;

std::atomic<void*> g_scratch_addr[kMaxDevices];

struct NaArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* kv_indptr;
  const int32_t* kv_indices;
  const int32_t* last_page_len;
  __nv_bfloat16* o;
  float* lse;
  float* part_o;     // [batch, Hk, n_chunks, G, D]
  float* part_lse;   // [batch, Hk, n_chunks, G]
  int32_t Hq, Hk, G, P, shift, chunk, n_chunks;
  float scale;       // sm_scale * log2(e)
};

__device__ __forceinline__ int kv_len_of(const NaArgs& a, int b) {
  const int np = a.kv_indptr[b + 1] - a.kv_indptr[b];
  return np > 0 ? (np - 1) * a.P + a.last_page_len[b] : 0;
}

// One CTA: request blockIdx.z, kv head blockIdx.y, keys [chunk * blockIdx.x, ...),
// through the same attention body as the planned decode kernel.
template <int D>
__global__ void __launch_bounds__(decode::kThreads, 2) noalloc_decode_kernel(const __grid_constant__ NaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int b = blockIdx.z, g = blockIdx.y, c = blockIdx.x;
  const int kv_len = kv_len_of(a, b);
  const int kv_lo = c * a.chunk;
  if (c > 0 && kv_lo >= kv_len) return;  // this chunk holds no key; the merge does not read it
  // the last chunk takes every remaining key, so a kv_len above max_kv_len is still exact
  const int kv_hi = c == a.n_chunks - 1 ? kv_len : min(kv_len, kv_lo + a.chunk);
  const size_t row0 = (size_t)b * a.Hq + (size_t)g * a.G;  // first of the group's query / output rows
  decode::Job jb;
  jb.q = a.q + row0 * D;
  jb.k = a.k;
  jb.v = a.v;
  jb.pages = a.kv_indices + a.kv_indptr[b];
  jb.kv_lo = kv_lo;
  jb.kv_hi = kv_hi;
  jb.kv_head = g;
  jb.G = a.G;
  jb.Hk = a.Hk;
  jb.P = a.P;
  jb.shift = a.shift;
  jb.scale = a.scale;
  if (a.n_chunks > 1) {
    const size_t prow = (((size_t)b * a.Hk + g) * a.n_chunks + c) * a.G;
    jb.part_o = a.part_o + prow * D;
    jb.part_lse = a.part_lse + prow;
    jb.o = nullptr;
    jb.lse = nullptr;
  } else {
    jb.part_o = nullptr;
    jb.part_lse = nullptr;
    jb.o = a.o + row0 * D;
    jb.lse = a.lse ? a.lse + row0 : nullptr;
  }
  decode::attend<D, false>(smem, jb);
}

// One CTA per (request, kv head): merge the chunks that hold keys.
template <int D>
__global__ void __launch_bounds__(128) noalloc_merge_kernel(const __grid_constant__ NaArgs a) {
  const int b = blockIdx.y, g = blockIdx.x;
  const int kv_len = kv_len_of(a, b);
  const int nv = kv_len > 0 ? min(a.n_chunks, (kv_len + a.chunk - 1) / a.chunk) : 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int row = warp; row < a.G; row += 4) {
    const size_t base = (((size_t)b * a.Hk + g) * a.n_chunks) * a.G + row;
    float m = -INFINITY;
    for (int i = 0; i < nv; ++i) m = fmaxf(m, a.part_lse[base + (size_t)i * a.G]);
    const float mu = m == -INFINITY ? 0.f : m;
    float L = 0.f;
    for (int i = 0; i < nv; ++i) L += ex2(a.part_lse[base + (size_t)i * a.G] - mu);
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const size_t orow = (size_t)b * a.Hq + g * a.G + row;
    for (int d = lane; d < D; d += 32) {
      float acc = 0.f;
      for (int i = 0; i < nv; ++i) {
        const size_t prow = base + (size_t)i * a.G;
        acc += ex2(a.part_lse[prow] - mu) * a.part_o[prow * D + d];
      }
      a.o[orow * D + d] = __float2bfloat16_rn(acc * inv);
    }
    if (lane == 0 && a.lse) a.lse[orow] = L > 0.f ? mu + __log2f(L) : -INFINITY;
  }
}

template <int D>
cudaError_t launch(const NaArgs& a, int batch, cudaStream_t st) {
  constexpr size_t smem = decode::smem_bytes<D>();
  // all of the unified L1 / shared array as shared memory, so two CTAs fit per SM
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attrs_once((const void*)noalloc_decode_kernel<D>, (int)smem, configured, true);
  if (e != cudaSuccess) return e;
  noalloc_decode_kernel<D><<<dim3(a.n_chunks, a.Hk, batch), decode::kThreads, smem, st>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.n_chunks <= 1) return e;
  noalloc_merge_kernel<D><<<dim3(a.Hk, batch), 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace

}  // namespace pkv

using namespace pkv;

extern "C" pkv_status pkv_decode_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                         const int32_t* kv_indptr, const int32_t* kv_indices,
                                         const int32_t* kv_last_page_len, int32_t batch, int32_t num_qo_heads,
                                         int32_t num_kv_heads, int32_t head_dim, int32_t page_size,
                                         int32_t max_kv_len, float sm_scale, void* o, float* lse, void* stream) {
  if (batch < 0 || max_kv_len < 0) {
    set_last_error("pkv_decode_noalloc: batch and max_kv_len must be >= 0");
    return PKV_EINVAL;
  }
  if (batch == 0) return PKV_OK;
  if (!q || !k_cache || !v_cache || !kv_indptr || !kv_indices || !kv_last_page_len || !o) {
    set_last_error("pkv_decode_noalloc: NULL pointer");
    return PKV_EINVAL;
  }
  // The kernels read q, K and V with 16-byte copies and 4-byte loads and write
  // O in 2-byte and LSE in 4-byte stores: refuse misaligned pointers on the
  // host rather than fault on the device.
  auto aligned = [](const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) & (n - 1)) == 0; };
  if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(o, 16) ||
      !aligned(kv_indptr, 4) || !aligned(kv_indices, 4) || !aligned(kv_last_page_len, 4) ||
      (lse && !aligned(lse, 4))) {
    set_last_error("pkv_decode_noalloc: q, k_cache, v_cache and o must be 16-byte aligned, index arrays and lse 4-byte");
    return PKV_EINVAL;
  }
  if (num_qo_heads <= 0 || num_kv_heads <= 0 || num_qo_heads % num_kv_heads != 0) {
    set_last_error("pkv_decode_noalloc: num_qo_heads must be a positive multiple of num_kv_heads");
    return PKV_EINVAL;
  }
  const int G = num_qo_heads / num_kv_heads;
  if (G > kRowsMax || (head_dim != 64 && head_dim != 128)) {
    set_last_error("pkv_decode_noalloc: needs num_qo_heads / num_kv_heads <= 16 and head_dim 64 or 128");
    return PKV_EUNSUPPORTED;
  }
  // batch and kv heads are grid dimensions y and z of the launches (at most 65535 each)
  if (batch > 65535 || num_kv_heads > 65535) {
    set_last_error("pkv_decode_noalloc: batch and num_kv_heads must be at most 65535 per call");
    return PKV_EUNSUPPORTED;
  }
  if (page_size <= 0 || page_size > 256 || (page_size & (page_size - 1)) != 0) {
    set_last_error("pkv_decode_noalloc: page_size must be a power of two in [1, 256]");
    return PKV_EUNSUPPORTED;
  }
  if (!(sm_scale > 0.f) || !(sm_scale < INFINITY)) {
    set_last_error("pkv_decode_noalloc: sm_scale must be positive and finite");
    return PKV_EUNSUPPORTED;
  }
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    set_last_error("pkv_decode_noalloc: no current CUDA device (or device ordinal >= 64)");
    return PKV_ECUDA;
  }
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    cudaGetLastError();
    sms = 148;
  }
  // Split each (request, kv head) into enough chunks to give every SM about
  // four CTAs, but never below 256 keys per chunk.
  const int64_t pairs = (int64_t)batch * num_kv_heads;
  const int64_t want = (4 * (int64_t)sms + pairs - 1) / pairs;
  const int64_t by_len = (max_kv_len + 255) / 256;
  int64_t n_chunks = std::max<int64_t>(1, std::min(want, by_len));
  int64_t chunk = max_kv_len > 0 ? ((max_kv_len + n_chunks - 1) / n_chunks + 63) / 64 * 64 : 64;
  n_chunks = max_kv_len > 0 ? (max_kv_len + chunk - 1) / chunk : 1;
  NaArgs a{};
  if (n_chunks > 1) {
    const size_t lse_bytes = ((size_t)pairs * n_chunks * G * sizeof(float) + 255) / 256 * 256;
    const size_t need = lse_bytes + (size_t)pairs * n_chunks * G * head_dim * sizeof(float);
    if (need > kNoAllocScratchBytes) {
      set_last_error("pkv_decode_noalloc: this batch needs " + std::to_string(need) +
                     " bytes of split-KV scratch, above the fixed 16 MiB the entry point owns; "
                     "use pkv_plan_create / pkv_run with a caller-allocated workspace");
      return PKV_ENOSPACE;
    }
    void* base = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!base) {
      cudaError_t e = cudaGetSymbolAddress(&base, g_noalloc_scratch);
      if (e != cudaSuccess || !base) {
        cudaGetLastError();
        set_last_error(std::string("pkv_decode_noalloc: cudaGetSymbolAddress failed: ") + cudaGetErrorString(e));
        return PKV_ECUDA;
      }
      g_scratch_addr[dev].store(base, std::memory_order_release);
    }
    a.part_lse = static_cast<float*>(base);
    a.part_o = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + lse_bytes);
  }
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k_cache);
  a.v = static_cast<const __nv_bfloat16*>(v_cache);
  a.kv_indptr = kv_indptr;
  a.kv_indices = kv_indices;
  a.last_page_len = kv_last_page_len;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.Hq = num_qo_heads;
  a.Hk = num_kv_heads;
  a.G = G;
  a.P = page_size;
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  a.shift = shift;
  a.chunk = (int32_t)chunk;
  a.n_chunks = (int32_t)n_chunks;
  a.scale = (float)((double)sm_scale * 1.4426950408889634);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = head_dim == 128 ? launch<128>(a, batch, st) : launch<64>(a, batch, st);
  if (e != cudaSuccess) {
    set_last_error(std::string("pkv_decode_noalloc: launch: ") + cudaGetErrorString(e));
    return PKV_ECUDA;
  }
  return PKV_OK;
}
