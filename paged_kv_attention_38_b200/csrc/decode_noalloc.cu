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
// The kernels are a copy of the split-KV decode of decode_sm100.cu in which a
// CTA takes its (request, kv head, KV chunk) from blockIdx and reads the
// request's length from the device page table, instead of from an uploaded work
// list.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <string>

#include "pkv.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

// Largest scratch any call may use; calls that would need more are rejected.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

void set_last_error(const std::string& msg);  // api.cu

namespace {

constexpr int kThreads = 128;
constexpr int kStages = 3;
constexpr int kTile = 64;          // keys per pipeline stage
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

template <int D>
__device__ __forceinline__ uint32_t kv_off(int r, int ch) {
  return (uint32_t)(r * (D * 2) + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ int kv_len_of(const NaArgs& a, int b) {
  const int np = a.kv_indptr[b + 1] - a.kv_indptr[b];
  return np > 0 ? (np - 1) * a.P + a.last_page_len[b] : 0;
}

// One CTA: request blockIdx.z, kv head blockIdx.y, keys [chunk * blockIdx.x, ...).
template <int D>
__global__ void __launch_bounds__(kThreads, 2) noalloc_decode_kernel(const __grid_constant__ NaArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kTileBytes = kTile * D * 2;
  constexpr int kChunks = D / 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = blockIdx.z, g = blockIdx.y, c = blockIdx.x;
  const int kv_len = kv_len_of(a, b);
  const int kv_lo = c * a.chunk;
  if (c > 0 && kv_lo >= kv_len) return;  // this chunk holds no key; the merge does not read it
  // the last chunk takes every remaining key, so a kv_len above max_kv_len is still exact
  const int kv_hi = c == a.n_chunks - 1 ? kv_len : min(kv_len, kv_lo + a.chunk);
  const int page0 = a.kv_indptr[b];
  const int G = a.G, Hk = a.Hk, P = a.P, shift = a.shift;
  const int n = kv_hi > kv_lo ? (kv_hi - kv_lo + kTile - 1) / kTile : 0;
  const uint32_t sbase = smem_u32(smem);

  auto load_tile = [&](int j, int stage) {
    const uint32_t kdst = sbase + stage * 2 * kTileBytes;
    const uint32_t vdst = kdst + kTileBytes;
    for (int x = tid; x < kTile * kChunks; x += kThreads) {
      const int r = x / kChunks, ch = x % kChunks;
      const int pos = kv_lo + j * kTile + r;
      const bool ok = pos < kv_hi;
      size_t off = 0;
      if (ok) {
        const int page = __ldg(a.kv_indices + page0 + (pos >> shift));
        off = (((size_t)page * P + (pos & (P - 1))) * Hk + g) * D + ch * 8;
      }
      cp_async_16(kdst + kv_off<D>(r, ch), a.k + off, ok ? 16u : 0u);
      cp_async_16(vdst + kv_off<D>(r, ch), a.v + off, ok ? 16u : 0u);
    }
  };
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < n) load_tile(s, s);
    cp_async_commit();
  }
  uint32_t qa[D / 16][4];
  {
    const int r0 = lane >> 2, kq = (lane & 3) * 2;
    const __nv_bfloat16* qrow = a.q + ((size_t)b * a.Hq + g * G) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      auto ld = [&](int row, int col) -> uint32_t {
        if (row >= G) return 0u;
        return *reinterpret_cast<const uint32_t*>(qrow + (size_t)row * D + col);
      };
      qa[kk][0] = ld(r0, kk * 16 + kq);
      qa[kk][1] = ld(r0 + 8, kk * 16 + kq);
      qa[kk][2] = ld(r0, kk * 16 + kq + 8);
      qa[kk][3] = ld(r0 + 8, kk * 16 + kq + 8);
    }
  }
  float o_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  for (int j = 0; j < n; ++j) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (j + kStages - 1 < n) load_tile(j + kStages - 1, (j + kStages - 1) % kStages);
    cp_async_commit();
    const uint32_t kst = sbase + (j % kStages) * 2 * kTileBytes;
    const uint32_t vst = kst + kTileBytes;
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int mi = lane >> 3;
      const int row = warp * 16 + (lane & 7) + (mi >> 1) * 8;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kst + kv_off<D>(row, kk * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816(s[0], qa[kk], b0, b1);
        mma16816(s[1], qa[kk], b2, b3);
      }
    }
    const int key0 = kv_lo + j * kTile + warp * 16 + (lane & 3) * 2;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        s[nt][e] = (key0 + nt * 8 + (e & 1)) < kv_hi ? s[nt][e] * a.scale : -INFINITY;
    float mx0 = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
    float mx1 = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
    const float a0 = m0 == n0 ? 1.f : ex2(m0 - u0), a1 = m1 == n1 ? 1.f : ex2(m1 - u1);
    m0 = n0;
    m1 = n1;
    float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      s[nt][0] = ex2(s[nt][0] - u0);
      s[nt][1] = ex2(s[nt][1] - u0);
      s[nt][2] = ex2(s[nt][2] - u1);
      s[nt][3] = ex2(s[nt][3] - u1);
      rs0 += s[nt][0] + s[nt][1];
      rs1 += s[nt][2] + s[nt][3];
    }
    l0 = l0 * a0 + rs0;
    l1 = l1 * a1 + rs1;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o_acc[i][0] *= a0;
      o_acc[i][1] *= a0;
      o_acc[i][2] *= a1;
      o_acc[i][3] *= a1;
    }
    uint32_t pa[4];
    pa[0] = pack_bf16x2(s[0][0], s[0][1]);
    pa[1] = pack_bf16x2(s[0][2], s[0][3]);
    pa[2] = pack_bf16x2(s[1][0], s[1][1]);
    pa[3] = pack_bf16x2(s[1][2], s[1][3]);
    {
      const int mi = lane >> 3;
      const int row = warp * 16 + (lane & 7) + (mi & 1) * 8;
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vst + kv_off<D>(row, np * 2 + (mi >> 1)), b0, b1, b2, b3);
        mma16816(o_acc[np * 2], pa, b0, b1);
        mma16816(o_acc[np * 2 + 1], pa, b2, b3);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* so = reinterpret_cast<float*>(smem);
  float* sm_m = so + 4 * 16 * D;
  float* sm_l = sm_m + 4 * 16;
  {
    const int r0 = lane >> 2, c0 = (lane & 3) * 2;
    float* ow = so + warp * 16 * D;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      ow[r0 * D + i * 8 + c0] = o_acc[i][0];
      ow[r0 * D + i * 8 + c0 + 1] = o_acc[i][1];
      ow[(r0 + 8) * D + i * 8 + c0] = o_acc[i][2];
      ow[(r0 + 8) * D + i * 8 + c0 + 1] = o_acc[i][3];
    }
    if ((lane & 3) == 0) {
      sm_m[warp * 16 + r0] = m0;
      sm_m[warp * 16 + r0 + 8] = m1;
      sm_l[warp * 16 + r0] = l0;
      sm_l[warp * 16 + r0 + 8] = l1;
    }
  }
  __syncthreads();
  for (int e = tid; e < G * D; e += kThreads) {
    const int row = e / D, d = e % D;
    float mm = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mm = fmaxf(mm, sm_m[w * 16 + row]);
    const float mu = mm == -INFINITY ? 0.f : mm;
    float L = 0.f, acc = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const float wt = ex2(sm_m[w * 16 + row] - mu);
      L += wt * sm_l[w * 16 + row];
      acc += wt * so[(w * 16 + row) * D + d];
    }
    const float out = L > 0.f ? acc / L : 0.f;
    const float lse2 = L > 0.f ? mu + __log2f(L) : -INFINITY;
    if (a.n_chunks > 1) {
      const size_t prow = (((size_t)b * Hk + g) * a.n_chunks + c) * G + row;
      a.part_o[prow * D + d] = out;
      if (d == 0) a.part_lse[prow] = lse2;
    } else {
      const size_t orow = (size_t)b * a.Hq + g * G + row;
      a.o[orow * D + d] = __float2bfloat16_rn(out);
      if (d == 0 && a.lse) a.lse[orow] = lse2;
    }
  }
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
  const size_t pipe = (size_t)kStages * 2 * kTile * D * 2;
  const size_t comb = (size_t)4 * 16 * D * 4 + 2 * 4 * 16 * 4;
  const size_t smem = pipe > comb ? pipe : comb;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(noalloc_decode_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    // all of the unified L1 / shared array as shared memory, so two CTAs fit per SM
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(noalloc_decode_kernel<D>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  noalloc_decode_kernel<D><<<dim3(a.n_chunks, a.Hk, batch), kThreads, smem, st>>>(a);
  cudaError_t e = cudaGetLastError();
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
  if (num_qo_heads <= 0 || num_kv_heads <= 0 || num_qo_heads % num_kv_heads != 0) {
    set_last_error("pkv_decode_noalloc: num_qo_heads must be a positive multiple of num_kv_heads");
    return PKV_EINVAL;
  }
  const int G = num_qo_heads / num_kv_heads;
  if (G > kRowsMax || (head_dim != 64 && head_dim != 128)) {
    set_last_error("pkv_decode_noalloc: needs num_qo_heads / num_kv_heads <= 16 and head_dim 64 or 128");
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
