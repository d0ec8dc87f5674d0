// Merging attention states by their base-2 LSE.
//
// FlashInfer 0.7.4 documentation, "Attention States and Recursive Attention"
// and "Merge Attention States": the attention of a query over a union of
// disjoint key sets follows from each part's (O_i, LSE_i):
//   LSE = log2(sum_i 2^LSE_i),   O = sum_i 2^(LSE_i - LSE) O_i.
// The split-KV schedule (discussion #15, disable_split_kv) relies on it.
//
// One warp per (output row, 128-column segment): each lane reads every
// part's LSE (a handful of floats, cached), then 4 columns of every part.
// A task's rows and segments are spread over blockIdx.y as well, so a few
// tasks with many rows (MLA decode: 16 heads x 512 columns x ~10 parts) still
// give thousands of warps, and the loops over parts are unrolled so that a
// warp's loads of several parts are in flight together (one part per
// iteration waited a full memory latency per part). The reads are coalesced
// along the row and the data is read once, so the kernel is bound by HBM
// traffic of the partials (small next to the KV stream that produced them).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

namespace {

constexpr int kWarps = 4;

__device__ __forceinline__ float part_max(const float* lse, size_t stride, int num) {
  float m = -INFINITY;
#pragma unroll 8
  for (int i = 0; i < num; ++i) m = fmaxf(m, lse[i * stride]);
  return m;
}

// Split-KV partial slots -> final bf16 O and fp32 LSE of the plan's outputs.
__global__ void __launch_bounds__(kWarps * 32) merge_tasks_kernel(const MergeTask* __restrict__ tasks, LaunchGeom g,
                                                                  const ReqInfo* __restrict__ reqs,
                                                                  const float* __restrict__ part_o,
                                                                  const float* __restrict__ part_lse,
                                                                  __nv_bfloat16* __restrict__ o,
                                                                  float* __restrict__ lse) {
  const MergeTask t = tasks[blockIdx.x];
  const ReqInfo req = reqs[t.req];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int Dv = g.head_dim_v, G = g.group, R = g.part_rows;
  const size_t slot_stride = (size_t)R;
  const int segs = (Dv + 127) / 128;
  for (int item = blockIdx.y * kWarps + warp; item < t.rows * segs; item += gridDim.y * kWarps) {
    const int r = item / segs, seg = item - r * segs;
    const float* lp = part_lse + (size_t)t.slot0 * R + r;
    const float m = part_max(lp, slot_stride, t.num);
    const float mu = m == -INFINITY ? 0.f : m;
    float L = 0.f;
#pragma unroll 8
    for (int i = 0; i < t.num; ++i) L += ex2(lp[i * slot_stride] - mu);
    const float inv = L > 0.f ? 1.f / L : 0.f;
    const int pr = t.row0 + r;
    const size_t orow = (size_t)(req.q_start + pr / G) * g.num_qo_heads + t.kv_head * G + pr % G;
    const int d = seg * 128 + lane * 4;
    if (d < Dv) {
      const float* op = part_o + ((size_t)t.slot0 * R + r) * Dv + d;
      const size_t part_stride = (size_t)R * Dv;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
      for (int i = 0; i < t.num; ++i) {
        const float w = ex2(lp[i * slot_stride] - mu);
        const float4 x = *reinterpret_cast<const float4*>(op + i * part_stride);
        acc.x += w * x.x;
        acc.y += w * x.y;
        acc.z += w * x.z;
        acc.w += w * x.w;
      }
      uint2 packed;
      packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
      packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
      *reinterpret_cast<uint2*>(o + orow * Dv + d) = packed;
    }
    if (lane == 0 && seg == 0 && lse) lse[orow] = L > 0.f ? mu + __log2f(L) : -INFINITY;
  }
}

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
__device__ __forceinline__ void store(float* p, float x) { *p = x; }
__device__ __forceinline__ void store(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

// Two states -> one state (may alias the first input): fp32 in and out, or
// bf16 O in and out (the outputs of two attention runs, as in cascade
// attention); the LSE is fp32 either way.
template <typename T>
__global__ void merge_state_kernel(const T* o_a, const float* lse_a, const T* o_b, const float* lse_b,
                                   T* o_out, float* lse_out, int rows, int dim) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const float la = lse_a[warp], lb = lse_b[warp];
  const float m = fmaxf(la, lb);
  const float mu = m == -INFINITY ? 0.f : m;
  const float wa = ex2(la - mu), wb = ex2(lb - mu);
  const float L = wa + wb;
  const float fa = L > 0.f ? wa / L : 0.f, fb = L > 0.f ? wb / L : 0.f;
  const size_t base = (size_t)warp * dim;
  for (int d = lane; d < dim; d += 32) store(o_out + base + d, fa * to_f32(o_a[base + d]) + fb * to_f32(o_b[base + d]));
  __syncwarp();
  if (lane == 0) lse_out[warp] = L > 0.f ? mu + __log2f(L) : -INFINITY;
}

// `num` fp32 states -> bf16 O, fp32 LSE.
__global__ void merge_states_kernel(const float* o_parts, const float* lse_parts, int num, int rows, int dim,
                                    __nv_bfloat16* o_out, float* lse_out) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const size_t stride = (size_t)rows;
  const float m = part_max(lse_parts + warp, stride, num);
  const float mu = m == -INFINITY ? 0.f : m;
  float L = 0.f;
  for (int i = 0; i < num; ++i) L += ex2(lse_parts[i * stride + warp] - mu);
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int d = lane; d < dim; d += 32) {
    float acc = 0.f;
    for (int i = 0; i < num; ++i)
      acc += ex2(lse_parts[i * stride + warp] - mu) * o_parts[((size_t)i * rows + warp) * dim + d];
    o_out[(size_t)warp * dim + d] = __float2bfloat16_rn(acc * inv);
  }
  if (lane == 0) lse_out[warp] = L > 0.f ? mu + __log2f(L) : -INFINITY;
}

}  // namespace

cudaError_t launch_merge_tasks(const LaunchGeom& g, const DeviceView& dv, void* o, float* lse,
                               cudaStream_t stream) {
  if (g.num_merge == 0) return cudaSuccess;
  const int segs = (g.head_dim_v + 127) / 128;
  const dim3 grid(g.num_merge, (g.part_rows * segs + kWarps - 1) / kWarps);
  merge_tasks_kernel<<<grid, kWarps * 32, 0, stream>>>(dv.merges, g, dv.reqs, dv.part_o, dv.part_lse,
                                                       static_cast<__nv_bfloat16*>(o), lse);
  return cudaGetLastError();
}

cudaError_t launch_merge_state(const float* o_a, const float* lse_a, const float* o_b, const float* lse_b,
                               float* o_out, float* lse_out, int rows, int dim, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int warps_per_block = 8;
  merge_state_kernel<float><<<(rows + warps_per_block - 1) / warps_per_block, warps_per_block * 32, 0, stream>>>(
      o_a, lse_a, o_b, lse_b, o_out, lse_out, rows, dim);
  return cudaGetLastError();
}

cudaError_t launch_merge_state_bf16(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                                    void* o_out, float* lse_out, int rows, int dim, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int warps_per_block = 8;
  merge_state_kernel<__nv_bfloat16><<<(rows + warps_per_block - 1) / warps_per_block, warps_per_block * 32, 0,
                                      stream>>>(static_cast<const __nv_bfloat16*>(o_a), lse_a,
                                                static_cast<const __nv_bfloat16*>(o_b), lse_b,
                                                static_cast<__nv_bfloat16*>(o_out), lse_out, rows, dim);
  return cudaGetLastError();
}

cudaError_t launch_merge_states(const float* o_parts, const float* lse_parts, int num, int rows, int dim,
                                void* o_out, float* lse_out, cudaStream_t stream) {
  if (rows == 0) return cudaSuccess;
  const int warps_per_block = 8;
  merge_states_kernel<<<(rows + warps_per_block - 1) / warps_per_block, warps_per_block * 32, 0, stream>>>(
      o_parts, lse_parts, num, rows, dim, static_cast<__nv_bfloat16*>(o_out), lse_out);
  return cudaGetLastError();
}

}  // namespace pkv
