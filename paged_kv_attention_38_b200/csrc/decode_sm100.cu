// Split-KV paged decode (one query token per request), built for HBM bandwidth.
//
// What it computes: the same paged attention as prefill with qo_len = 1
// (FlashInfer 0.7.4 documentation, flashinfer.decode; page table as in
// flashinfer-trace discussion #15, "Notes on fa3_gqa_prefill_v1"). One CTA
// handles one work unit of the plan, a (request, kv head, KV chunk); the
// `group` query heads that share the kv head share every K/V byte it loads, so
// K and V are read from HBM once. Chunks of a split request write fp32 partial
// states into the plan's workspace, which the merge kernel combines by their
// base-2 LSE ("Merge Attention States"). The attention over a chunk is
// decode::attend (decode_core.cuh): a 3-stage cp.async ring of 64-key K/V
// tiles, mma.sync for the small contractions, two CTAs per SM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "decode_core.cuh"
#include "launch_util.h"
#include "pkv_internal.h"

namespace pkv {

namespace {

struct Args {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* kv_indices;
  __nv_bfloat16* o;
  float* lse;
  LaunchGeom g;
  DeviceView dv;
};

template <int D, bool kHnd>
__global__ void __launch_bounds__(decode::kThreads, 2) decode_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const WorkUnit unit = a.dv.units[blockIdx.x];
  const ReqInfo req = a.dv.reqs[unit.req];
  const int G = a.g.group;
  // the group's G query heads (and output rows) are consecutive rows of D
  const size_t row0 = (size_t)req.q_start * a.g.num_qo_heads + (size_t)unit.kv_head * G;
  decode::Job jb;
  jb.q = a.q + row0 * D;
  jb.k = a.k;
  jb.v = a.v;
  jb.pages = a.kv_indices + req.page0;
  jb.kv_lo = unit.kv_lo;
  jb.kv_hi = unit.kv_hi;
  jb.kv_head = unit.kv_head;
  jb.G = G;
  jb.Hk = a.g.num_kv_heads;
  jb.P = a.g.page_size;
  jb.shift = a.g.page_shift;
  jb.scale = a.g.sm_scale_log2;
  if (unit.partial >= 0) {
    const size_t prow = (size_t)unit.partial * kDecodeRows;
    jb.part_o = a.dv.part_o + prow * D;
    jb.part_lse = a.dv.part_lse + prow;
    jb.o = nullptr;
    jb.lse = nullptr;
  } else {
    jb.part_o = nullptr;
    jb.part_lse = nullptr;
    jb.o = a.o + row0 * D;
    jb.lse = a.lse ? a.lse + row0 : nullptr;
  }
  decode::attend<D, kHnd>(smem, jb);
}

template <int D, bool kHnd>
cudaError_t launch(const Args& a, cudaStream_t stream) {
  constexpr size_t smem = decode::smem_bytes<D>();
  auto kern = decode_kernel<D, kHnd>;
  // all of the unified L1 / shared array as shared memory, so two CTAs fit per SM
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attrs_once((const void*)kern, (int)smem, configured, true);
  if (e != cudaSuccess) return e;
  kern<<<a.g.num_units, decode::kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices, const void* q,
                          const void* k, const void* v, void* o, float* lse, cudaStream_t stream) {
  if (g.num_units == 0) return cudaSuccess;
  Args a{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
         static_cast<const __nv_bfloat16*>(v), kv_indices, static_cast<__nv_bfloat16*>(o), lse, g, dv};
  const bool hnd = g.kv_layout == 1;
  if (g.head_dim == 128) return hnd ? launch<128, true>(a, stream) : launch<128, false>(a, stream);
  if (g.head_dim == 64) return hnd ? launch<64, true>(a, stream) : launch<64, false>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pkv
