// Paged causal GQA prefill on sm_100a tensor cores (tcgen05, accumulators in TMEM).
//
// What it computes (flashinfer-trace discussion #15, definition
// gqa_paged_prefill_causal_h16_kv1_d128_ps64 and "Notes on fa3_gqa_prefill_v1";
// FlashInfer 0.2 release, "FlashAttention-3 template with block/vector
// sparsity"): for each work unit (request, kv head, 128 packed query rows,
// KV range), O = softmax(sm_scale Q K^T + causal mask) V over the keys the
// page table lists, plus the base-2 LSE of every row. The K/V rows of a tile
// are gathered page by page through kv_indices, so page_size = 1 (vector
// sparsity) and page_size = 64 run the same code; only the gather differs
// from dense attention.
//
// CTA layout (288 threads, one work unit per CTA):
//   warps 0-3  softmax + epilogue. Thread i owns query row i = TMEM lane i.
//   warp  4    TMEM allocator and MMA issuer (one lane issues tcgen05.mma).
//   warps 5-8  producer: cp.async gather of Q once, then K/V tiles of 128 keys
//              into a 2-stage ring, 16-byte copies, 128-byte swizzled rows.
// TMEM (512 columns): S double buffer at columns [0,128) and [128,256), O at
// [256, 256 + D). P goes through shared memory as the A operand of P.V.
//
// Per KV tile j the MMA warp issues S_j = Q K_j^T (into S buffer j%2) before
// O += P_{j-1} V_{j-1}, so the softmax of tile j overlaps the P.V of tile j-1.
// Online softmax runs in the base-2 domain: s' = s * sm_scale * log2(e),
// p = 2^(s' - m); O is rescaled in TMEM only when a row's max grows.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

namespace {

constexpr int kThreads = 288;
constexpr int kSoftmaxThreads = 128;
constexpr int kProducerThreads = 128;
constexpr int kProducerWarp0 = 5;
constexpr int kMmaWarp = 4;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;

// Byte offset of 16-byte chunk `ch` (of row length D/8 chunks) of row `r` in a
// [128 x D] bf16 tile stored as D/64 column blocks of [128 rows x 128 B] with
// the 128-byte swizzle (chunk index XOR row % 8).
__device__ __forceinline__ uint32_t tile_off(int r, int ch) {
  return (uint32_t)((ch >> 3) * (kBlockM * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int D>
struct __align__(1024) Smem {
  __nv_bfloat16 q[kBlockM * D];
  __nv_bfloat16 k[kStages][kBlockN * D];
  __nv_bfloat16 v[kStages][kBlockN * D];
  __nv_bfloat16 p[kBlockM * kBlockN];
  uint64_t q_full;
  uint64_t k_full[kStages];
  uint64_t v_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full;
  uint64_t o_done;
  uint32_t tmem_base;
  int abort_flag;
};

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

template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ Args a) {
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  const WorkUnit unit = a.dv.units[blockIdx.x];
  const ReqInfo req = a.dv.reqs[unit.req];
  const int G = a.g.group;
  const int n_tiles = (unit.kv_hi - unit.kv_lo + kBlockN - 1) / kBlockN;

  if (tid == 0) {
    mbar_init(&sm.q_full, kProducerThreads);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.k_full[s], kProducerThreads);
      mbar_init(&sm.v_full[s], kProducerThreads);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], kSoftmaxThreads);
    }
    mbar_init(&sm.p_full, kSoftmaxThreads);
    mbar_init(&sm.o_done, 1);
    sm.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  WaitCtx wc{&sm.abort_flag, a.dv.status};

  if (warp >= kProducerWarp0) {
    // ------------------------------------------------------------ producer
    const int pt = tid - kProducerWarp0 * 32;
    constexpr int kChunks = D / 8;  // 16-byte chunks per row
    const size_t head_stride_q = (size_t)a.g.num_qo_heads * D;
    // Q tile: packed row r -> token q_start + (row0 + r) / G, head kv_head*G + (row0 + r) % G
    for (int c = pt; c < kBlockM * kChunks; c += kProducerThreads) {
      const int r = c / kChunks, ch = c % kChunks;
      const bool ok = r < unit.rows;
      const __nv_bfloat16* src = a.q;
      if (ok) {
        const int pr = unit.row0 + r;
        const int t = req.q_start + pr / G;
        const int h = unit.kv_head * G + pr % G;
        src = a.q + (size_t)t * head_stride_q + (size_t)h * D + ch * 8;
      }
      cp_async_16(smem_u32(sm.q) + tile_off(r, ch), src, ok ? 16u : 0u);
    }
    cp_async_commit();
    const int P = a.g.page_size, shift = a.g.page_shift, Hk = a.g.num_kv_heads;
    auto load_kv = [&](const __nv_bfloat16* base, __nv_bfloat16* dst, int j) {
      for (int c = pt; c < kBlockN * kChunks; c += kProducerThreads) {
        const int r = c / kChunks, ch = c % kChunks;
        const int pos = unit.kv_lo + j * kBlockN + r;
        const bool ok = pos < unit.kv_hi;
        const __nv_bfloat16* src = base;
        if (ok) {
          const int page = __ldg(a.kv_indices + req.page0 + (pos >> shift));
          const int slot = pos & (P - 1);
          src = base + (((size_t)page * P + slot) * Hk + unit.kv_head) * D + ch * 8;
        }
        cp_async_16(smem_u32(dst) + tile_off(r, ch), src, ok ? 16u : 0u);
      }
      cp_async_commit();
    };
    // Each group is signalled once the next one is in flight (wait_group 1),
    // after this thread's fence.proxy.async makes its copies visible to the
    // tensor core.
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      if (j >= kStages) mbar_wait(&sm.kv_empty[s], ((j >> 1) - 1) & 1, wc);
      load_kv(a.k, sm.k[s], j);
      cp_async_wait<1>();
      fence_proxy_async_smem();
      if (j == 0) mbar_arrive(&sm.q_full);
      else mbar_arrive(&sm.v_full[(j - 1) & 1]);
      load_kv(a.v, sm.v[s], j);
      cp_async_wait<1>();
      fence_proxy_async_smem();
      mbar_arrive(&sm.k_full[s]);
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();
    if (n_tiles > 0) mbar_arrive(&sm.v_full[(n_tiles - 1) & 1]);
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kBlockM, D, true);
      const uint32_t q_addr = smem_u32(sm.q);
      const uint32_t p_addr = smem_u32(sm.p);
      const uint32_t o_tmem = tmem + 256;
      auto issue_pv = [&](int jj) {
        const int sp = jj & 1;
        mbar_wait(&sm.p_full, jj & 1, wc);
        mbar_wait(&sm.v_full[sp], (jj >> 1) & 1, wc);
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm.v[sp]);
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk) {
          const uint64_t da = sdesc_sw128(p_addr + (kk >> 2) * (kBlockM * 128) + (kk & 3) * 32, 16, 1024);
          const uint64_t db = sdesc_sw128(v_addr + kk * 16 * 128, kBlockN * 128, 1024);
          umma_bf16(o_tmem, da, db, idesc_o, (jj > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&sm.o_done);
        umma_commit(&sm.kv_empty[sp]);
      };
      mbar_wait(&sm.q_full, 0, wc);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        mbar_wait(&sm.k_full[s], (j >> 1) & 1, wc);
        if (j >= 2) mbar_wait(&sm.s_free[s], ((j >> 1) - 1) & 1, wc);
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.k[s]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBlockM * 128) + (kk & 3) * 32;
          umma_bf16(tmem + s * kBlockN, sdesc_sw128(q_addr + off, 16, 1024),
                    sdesc_sw128(k_addr + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit(&sm.s_full[s]);
        if (j >= 1) issue_pv(j - 1);
      }
      issue_pv(n_tiles - 1);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int r = tid;  // query row == TMEM lane
    const bool row_ok = r < unit.rows;
    const int pr = unit.row0 + (row_ok ? r : 0);
    const int t = pr / G;  // token index within the request
    int limit = unit.kv_hi;  // exclusive bound on key position for this row
    if (a.g.causal) limit = min(limit, t + req.kv_len - req.qo_len + 1);
    const float scale = a.g.sm_scale_log2;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t o_tmem = lane_base + 256;
    float m = -INFINITY, l = 0.f;
    const uint32_t p_addr = smem_u32(sm.p);
    float sv[kBlockN];
    for (int j = 0; j < n_tiles; ++j) {
      const int s = j & 1;
      mbar_wait(&sm.s_full[s], (j >> 1) & 1, wc);
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < kBlockN; c += 32) tmem_ld32(lane_base + s * kBlockN + c, sv + c);
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&sm.s_free[s]);
      const int kv0 = unit.kv_lo + j * kBlockN;
      float mx = -INFINITY;
      if (kv0 + kBlockN <= limit) {
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) {
          sv[c] *= scale;
          mx = fmaxf(mx, sv[c]);
        }
      } else {
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) {
          sv[c] = (kv0 + c < limit) ? sv[c] * scale : -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
      }
      const float m_new = fmaxf(m, mx);
      const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = (m == m_new) ? 1.f : ex2(m - m_use);
      float rs = 0.f;
#pragma unroll
      for (int c = 0; c < kBlockN; ++c) {
        sv[c] = ex2(sv[c] - m_use);
        rs += sv[c];
      }
      l = l * alpha + rs;
      m = m_new;
      if (j > 0) {
        mbar_wait(&sm.o_done, (j - 1) & 1, wc);
        tc_fence_after();
      }
      // P_j (bf16, swizzled K-major rows) -> shared memory
#pragma unroll
      for (int ch = 0; ch < kBlockN / 8; ++ch) {
        uint4 w;
        w.x = pack_bf16x2(sv[ch * 8 + 0], sv[ch * 8 + 1]);
        w.y = pack_bf16x2(sv[ch * 8 + 2], sv[ch * 8 + 3]);
        w.z = pack_bf16x2(sv[ch * 8 + 4], sv[ch * 8 + 5]);
        w.w = pack_bf16x2(sv[ch * 8 + 6], sv[ch * 8 + 7]);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_addr + tile_off(r, ch)), "r"(w.x),
                     "r"(w.y), "r"(w.z), "r"(w.w)
                     : "memory");
      }
      fence_proxy_async_smem();
      if (j > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
        float ov[32];
#pragma unroll
        for (int c = 0; c < D; c += 32) {
          tmem_ld32(o_tmem + c, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] *= alpha;
          tmem_st32(o_tmem + c, ov);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&sm.p_full);
    }
    // ---------------------------------------------------------- epilogue
    if (n_tiles > 0) {
      mbar_wait(&sm.o_done, (n_tiles - 1) & 1, wc);
      tc_fence_after();
    }
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const float lse2 = l > 0.f ? m + __log2f(l) : -INFINITY;
    const int tok = req.q_start + t;
    const int h = unit.kv_head * G + pr % G;
    const int Dv = D;
    if (unit.partial >= 0) {
      float* dst = a.dv.part_o + ((size_t)unit.partial * kBlockM + r) * Dv;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        if (n_tiles > 0) {
          tmem_ld32(o_tmem + c, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0.f;
        }
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4*>(dst + c + i) =
                make_float4(ov[i] * inv_l, ov[i + 1] * inv_l, ov[i + 2] * inv_l, ov[i + 3] * inv_l);
        }
      }
      if (row_ok) a.dv.part_lse[(size_t)unit.partial * kBlockM + r] = lse2;
    } else {
      __nv_bfloat16* dst = a.o + ((size_t)tok * a.g.num_qo_heads + h) * Dv;
#pragma unroll
      for (int c = 0; c < D; c += 32) {
        float ov[32];
        if (n_tiles > 0) {
          tmem_ld32(o_tmem + c, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = 0.f;
        }
        if (row_ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 8) {
            uint4 w;
            w.x = pack_bf16x2(ov[i + 0] * inv_l, ov[i + 1] * inv_l);
            w.y = pack_bf16x2(ov[i + 2] * inv_l, ov[i + 3] * inv_l);
            w.z = pack_bf16x2(ov[i + 4] * inv_l, ov[i + 5] * inv_l);
            w.w = pack_bf16x2(ov[i + 6] * inv_l, ov[i + 7] * inv_l);
            *reinterpret_cast<uint4*>(dst + c + i) = w;
          }
        }
      }
      if (row_ok && a.lse) a.lse[(size_t)tok * a.g.num_qo_heads + h] = lse2;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
cudaError_t launch(const Args& a, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<D>) + 1024;
  auto kern = prefill_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<a.g.num_units, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_prefill(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices, const void* q,
                           const void* k, const void* v, void* o, float* lse, cudaStream_t stream) {
  if (g.num_units == 0) return cudaSuccess;
  Args a{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
         static_cast<const __nv_bfloat16*>(v), kv_indices, static_cast<__nv_bfloat16*>(o), lse, g, dv};
  if (g.head_dim == 128) return launch<128>(a, stream);
  if (g.head_dim == 64) return launch<64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pkv
