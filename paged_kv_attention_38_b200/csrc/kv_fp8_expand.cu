// FP8 E4M3 KV pages -> bf16 pages, for prefill over a quantised KV cache.
//
// What it serves: the per-head-scale quantised KV cache ("[Roadmap] FlashInfer
// v0.2 to v0.3", milestone "Per Head Scale Quantized KV-Cache") read by a
// prefill plan. Prefill is bound by the tensor cores, whose kind::f16 MMAs
// take A and B of one 16-bit type, so the page codes become bf16 operands
// before the attention kernel runs. Every E4M3 value is exact in bf16 (4
// significant bits, exponents 2^-9 .. 2^8), so the copy holds the codes'
// values exactly; the per-kv-head scales stay out of it and are applied by
// the prefill kernel (K's to the scores, V's to the output).
//
// One CTA per entry e of the batch's page table: it writes the page's codes as
// bf16 to entry e of a compact copy ([entries][page_size][Hk][D], NHD) and
// entry e of an identity page table, so the prefill kernel runs on the copy
// with the plan's own schedule. Slots past the request's last key are written
// as zeros: the prefill kernel reads whole pages and only masks their scores,
// and a NaN code there would otherwise reach the output through 0 * NaN.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "pkv_internal.h"

namespace pkv {

namespace {

constexpr int kThreads = 256;

struct ExpandArgs {
  const uint8_t* k_codes;
  const uint8_t* v_codes;
  const int32_t* kv_indices;
  const ReqInfo* reqs;
  __nv_bfloat16* k_out;
  __nv_bfloat16* v_out;
  int32_t* idx_out;
  int32_t batch, page_size, num_kv_heads, head_dim;
};

// Eight codes (bytes of w, low first) -> eight bf16, exact.
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 w) {
  uint32_t out[4];
  const uint32_t src[2] = {w.x, w.y};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t pair = (uint16_t)(src[i >> 1] >> ((i & 1) * 16));
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(pair));
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x, f.y);
    out[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(kThreads) kv_fp8_expand_kernel(const __grid_constant__ ExpandArgs a) {
  const int e = blockIdx.x;  // page-table entry
  // the request whose pages hold entry e: the last one with page0 <= e
  int lo = 0, hi = a.batch - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (a.reqs[mid].page0 <= e) lo = mid;
    else hi = mid - 1;
  }
  const ReqInfo req = a.reqs[lo];
  const int first_key = (e - req.page0) * a.page_size;  // the request's key held by slot 0 of this page
  const int page = a.kv_indices[e];
  if (threadIdx.x == 0) a.idx_out[e] = e;
  const int row_chunks = a.num_kv_heads * a.head_dim / 8;  // 8 codes per chunk, per slot
  const int chunks = a.page_size * row_chunks;
  const size_t in0 = (size_t)page * chunks, out0 = (size_t)e * chunks;
  const uint2* kin = reinterpret_cast<const uint2*>(a.k_codes) + in0;
  const uint2* vin = reinterpret_cast<const uint2*>(a.v_codes) + in0;
  uint4* kout = reinterpret_cast<uint4*>(a.k_out) + out0;
  uint4* vout = reinterpret_cast<uint4*>(a.v_out) + out0;
  for (int c = threadIdx.x; c < chunks; c += kThreads) {
    const bool live = first_key + c / row_chunks < req.kv_len;
    uint4 kb = make_uint4(0u, 0u, 0u, 0u), vb = kb;
    if (live) {
      kb = e4m3x8_to_bf16x8(__ldg(kin + c));
      vb = e4m3x8_to_bf16x8(__ldg(vin + c));
    }
    kout[c] = kb;
    vout[c] = vb;
  }
}

}  // namespace

cudaError_t launch_kv_fp8_expand(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices,
                                 int32_t num_entries, const void* k_codes, const void* v_codes, void* k_out,
                                 void* v_out, int32_t* idx_out, cudaStream_t stream) {
  if (num_entries <= 0) return cudaSuccess;
  if (g.head_dim % 8 != 0) return cudaErrorInvalidValue;
  ExpandArgs a{static_cast<const uint8_t*>(k_codes), static_cast<const uint8_t*>(v_codes), kv_indices, dv.reqs,
               static_cast<__nv_bfloat16*>(k_out), static_cast<__nv_bfloat16*>(v_out), idx_out,
               g.num_reqs, g.page_size, g.num_kv_heads, g.head_dim};
  kv_fp8_expand_kernel<<<(unsigned)num_entries, kThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace pkv
