// Absorbed-MLA paged prefill on sm_100a tensor cores.
//
// What it computes (FlashInfer 0.2 release, "Fused MLA decode kernel" and its
// matrix-absorption trick; definition mla_paged_prefill_causal_h16_ckv512_kpe64_ps1
// in flashinfer-trace discussion #15): all H query heads share one latent KV
// row per token, the compressed ckv (512) and the rope key kpe (64). With the
// projections absorbed into the query and output,
//   s_j = sm_scale * (q_nope . ckv_j + q_pe . kpe_j),   o = sum_j softmax(s)_j ckv_j,
// i.e. attention with a 576-wide key [ckv | kpe] and a 512-wide value ckv.
// Output O (bf16, 512 per head) and the base-2 LSE per (token, head).
//
// Shape choices for B200. A 128-row tile's 128 x 512 fp32 output alone would
// fill all 512 TMEM columns, and a 128 x 576 bf16 query tile (144 KB) leaves no
// room in shared memory for a double-buffered key tile. So a CTA takes 64
// packed (token, head) rows and 64-key tiles, and runs M = 64 MMAs:
//   TMEM  O rows x latent[0,256)   lanes 16q + [0,16)  (q = sub-partition), cols [0,256)
//         O rows x latent[256,512) lanes 16q + [16,32),                     cols [0,256)
//         S (double buffer)        lanes 16q + [0,16),                      cols [256,320), [320,384)
//   (a 64-row accumulator uses half of each 32-lane sub-partition; the two
//   latent halves of O sit in the two halves, so a warp rescales both with one
//   32x32b load/store over columns [0,256) without touching S.)
//   SMEM  Q 64 x 576 (72 KB), a 2-stage ring of 64 x 576 latent rows (K and V
//   at once: V is the ckv part of the same rows), P 64 x 64 (8 KB).
// Both MMAs read their operands from shared memory. The kernel is persistent:
// one CTA per SM runs a host-planned list of units, its barrier phases running
// on across units, so the next unit's Q and latent rows stream in while the
// previous unit finishes. Warps: 0-3 softmax and
// epilogue (lanes 0-15 own S rows and the low O half, lanes 16-31 the high O
// half of the same rows), 4 TMEM allocator + MMA issuer, 5-8 cp.async gather
// of Q and of the latent rows through the page table.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "launch_util.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

namespace {

constexpr int kRows = kMlaUnitRows;  // 64
constexpr int kN = 64;               // keys per tile
constexpr int kDc = 512;
constexpr int kDr = 64;
constexpr int kDqk = kDc + kDr;      // 576
constexpr int kBlocks = kDqk / 64;   // 9 column blocks of 64 (128-byte rows)
constexpr int kBlockBytes = kRows * 128;  // one [64 rows x 64] bf16 block: 8 KB
constexpr int kThreads = 288;
constexpr int kMmaWarp = 4;
constexpr int kProdWarp0 = 5;
constexpr int kProdThreads = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 256;
constexpr float kRescaleThreshold = 8.0f;
static_assert(kN == kRows, "one block shape for Q, latent rows and P");

// Byte offset of 16-byte chunk `ch` (0..71 across the 576-wide row) of row `r`
// in a [64 x 576] tile held as 9 column blocks of [64 rows x 128 B], 128-byte swizzle.
__device__ __forceinline__ uint32_t blk_off(int r, int ch) {
  return (uint32_t)((ch >> 3) * kBlockBytes + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

struct __align__(1024) Smem {
  __nv_bfloat16 q[kBlocks * kRows * 64];
  __nv_bfloat16 kv[2][kBlocks * kN * 64];
  __nv_bfloat16 p[kRows * kN];
  uint64_t q_full;
  uint64_t q_empty;  // the unit's last QK^T MMAs are done: Q may be overwritten
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full;
  uint64_t o_done;
  uint64_t o_final;
  int32_t rowsrc[2][kN];  // pool slot of each latent row of the tile in each stage, -1 = zero fill
  uint32_t tmem_base;
  int abort_flag;
};

struct Args {
  const __nv_bfloat16* q_nope;
  const __nv_bfloat16* q_pe;
  const __nv_bfloat16* ckv;
  const __nv_bfloat16* kpe;
  const int32_t* kv_indices;
  __nv_bfloat16* o;
  float* lse;
  LaunchGeom g;
  DeviceView dv;
};

__global__ void __launch_bounds__(kThreads, 1) mla_kernel(const __grid_constant__ Args a) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // Persistent: CTA b runs units [cta_ptr[b], cta_ptr[b + 1]); barrier phases
  // run on across units (counters of latent tiles and of units with keys).
  const int u_begin = a.dv.cta_ptr[blockIdx.x];
  const int u_end = a.dv.cta_ptr[blockIdx.x + 1];
  const int H = a.g.num_qo_heads;
  auto tiles_of = [](const WorkUnit& u) { return (u.kv_hi - u.kv_lo + kN - 1) / kN; };

  if (tid == 0) {
    mbar_init(&sm.q_full, kProdThreads);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.kv_full[s], kProdThreads);
      mbar_init(&sm.kv_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_free[s], 128);
    }
    mbar_init(&sm.p_full, 128);
    mbar_init(&sm.o_done, 1);
    mbar_init(&sm.o_final, 1);
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

  if (warp >= kProdWarp0) {
    // ================================================================ producer
    const int pt = tid - kProdWarp0 * 32;
    constexpr int kChunks = kDqk / 8;  // 72 16-byte chunks per 576-wide row
    const int P = a.g.page_size, shift = a.g.page_shift;
    int g = 0;   // latent tiles loaded by this CTA (stage g & 1)
    int uq = 0;  // units with keys whose Q was loaded
    for (int ui = u_begin; ui < u_end; ++ui) {
      const WorkUnit unit = a.dv.units[ui];
      const int n_tiles = tiles_of(unit);
      if (n_tiles == 0) continue;
      const ReqInfo req = a.dv.reqs[unit.req];
      // Q, once the previous unit's QK^T MMAs have read the old one
      if (uq > 0) mbar_wait(&sm.q_empty, (uq - 1) & 1, wc);
      for (int c = pt; c < kRows * kChunks; c += kProdThreads) {
        const int r = c / kChunks, ch = c % kChunks;
        const bool ok = r < unit.rows;
        const __nv_bfloat16* src = a.q_nope;
        if (ok) {
          const int pr = unit.row0 + r;
          const size_t row = (size_t)(req.q_start + pr / H) * H + pr % H;
          src = ch < kDc / 8 ? a.q_nope + row * kDc + ch * 8 : a.q_pe + row * kDr + (ch - kDc / 8) * 8;
        }
        cp_async_16(smem_u32(sm.q) + blk_off(r, ch), src, ok ? 16u : 0u);
      }
      cp_async_arrive_noinc(&sm.q_full);
      ++uq;
      // Latent tiles: the page lookups of a tile are done once (one row per
      // thread) into shared memory; then each thread copies a fixed 16-byte
      // column of every other row: ckv columns 0..63 (two rows per pass), kpe
      // columns 64..71 (sixteen rows per pass).
      for (int j = 0; j < n_tiles; ++j, ++g) {
        const int st = g & 1;
        if (g >= 2) mbar_wait(&sm.kv_empty[st], ((g >> 1) - 1) & 1, wc);
        if (pt < kN) {
          const int pos = unit.kv_lo + j * kN + pt;
          sm.rowsrc[st][pt] = pos < unit.kv_hi ? __ldg(a.kv_indices + req.page0 + (pos >> shift)) * P + (pos & (P - 1)) : -1;
        }
        named_bar_sync(1, kProdThreads);
        const uint32_t dst = smem_u32(sm.kv[st]);
        {
          const int ch = pt & 63;
          const uint32_t col = (uint32_t)((ch >> 3) * kBlockBytes + ((ch & 7) << 4));
          for (int r = pt >> 6; r < kN; r += 2) {
            const int src = sm.rowsrc[st][r];
            const __nv_bfloat16* gp = src >= 0 ? a.ckv + (size_t)src * kDc + ch * 8 : a.ckv;
            cp_async_16(dst + r * 128 + (col ^ ((r & 7) << 4)), gp, src >= 0 ? 16u : 0u);
          }
        }
        {
          const int ch = pt & 7;
          const uint32_t col = (uint32_t)(8 * kBlockBytes + (ch << 4));
          for (int r = pt >> 3; r < kN; r += 16) {
            const int src = sm.rowsrc[st][r];
            const __nv_bfloat16* gp = src >= 0 ? a.kpe + (size_t)src * kDr + ch * 8 : a.kpe;
            cp_async_16(dst + r * 128 + (col ^ ((r & 7) << 4)), gp, src >= 0 ? 16u : 0u);
          }
        }
        cp_async_arrive_noinc(&sm.kv_full[st]);
      }
    }
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    // The whole warp runs the loop (waits, descriptor arithmetic); one elected
    // lane (always lane 0) issues each tcgen05.mma / commit. Issued from a
    // single divergent lane, each MMA cost about 100 cycles of issue time, more
    // than its M = 64 execution time.
    constexpr uint32_t idesc_s = idesc_bf16_f32(kRows, kN, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(kRows, 256, true);
    const uint64_t dq = sdesc_sw128(smem_u32(sm.q), 16, 1024);
    const uint64_t dp = sdesc_sw128(smem_u32(sm.p), 16, 1024);
    uint64_t dk[2], dvv[2];
    for (int s = 0; s < 2; ++s) {
      dk[s] = sdesc_sw128(smem_u32(sm.kv[s]), 16, 1024);
      dvv[s] = sdesc_sw128(smem_u32(sm.kv[s]), kBlockBytes, 1024);
    }
    // O += P V for the CTA's latent tile gg; `first`: the unit's first tile
    auto issue_pv = [&](int gg, bool first) {
      const int st = gg & 1;
      mbar_wait(&sm.p_full, gg & 1, wc);
      fence_proxy_async_smem();
      tc_fence_after();
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        const uint32_t d = tmem + (nh ? (16u << 16) : 0u);
#pragma unroll
        for (int kk = 0; kk < kN / 16; ++kk)
          umma_bf16_ss_elect(d, dp + ((kk * 32) >> 4), dvv[st] + ((4 * nh * kBlockBytes + kk * 16 * 128) >> 4),
                             idesc_o, (!first || kk > 0) ? 1u : 0u);
      }
      umma_commit_elect(&sm.o_done);
      umma_commit_elect(&sm.kv_empty[st]);
    };
    int g = 0;   // latent tiles of this CTA: stage g & 1 and the per-tile phases
    int uq = 0;  // units with keys: q_full / q_empty / o_final phases
    for (int ui = u_begin; ui < u_end; ++ui) {
      const int n_tiles = tiles_of(a.dv.units[ui]);
      if (n_tiles == 0) continue;
      mbar_wait(&sm.q_full, uq & 1, wc);
      for (int j = 0; j < n_tiles; ++j, ++g) {
        const int st = g & 1;
        mbar_wait(&sm.kv_full[st], (g >> 1) & 1, wc);
        if (g >= 2) mbar_wait(&sm.s_free[st], ((g >> 1) - 1) & 1, wc);
        fence_proxy_async_smem();  // cp.async rows were written through the generic proxy
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kDqk / 16; ++kk) {
          const uint32_t off = ((kk >> 2) * kBlockBytes + (kk & 3) * 32) >> 4;
          umma_bf16_ss_elect(tmem + kSCol + st * kN, dq + off, dk[st] + off, idesc_s, kk > 0 ? 1u : 0u);
        }
        umma_commit_elect(&sm.s_full[st]);
        if (j + 1 == n_tiles) umma_commit_elect(&sm.q_empty);  // the unit's last QK^T is issued
        if (j >= 1) issue_pv(g - 1, j == 1);
      }
      issue_pv(g - 1, n_tiles == 1);
      umma_commit_elect(&sm.o_final);
      ++uq;
    }
    // no MMA may still run when TMEM is released
    if (uq > 0) mbar_drain(&sm.o_final, (uq - 1) & 1);
    __syncwarp();
  } else {
    // ================================================================ softmax
    const bool s_owner = lane < 16;
    const int row = warp * 16 + (lane & 15);  // row of the unit this thread's S / O half belongs to
    const float scale = a.g.sm_scale_log2;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t p_addr = smem_u32(sm.p);
    int g = 0, uq = 0;  // latent tiles and units with keys done by this CTA
    for (int ui = u_begin; ui < u_end; ++ui) {
      const WorkUnit unit = a.dv.units[ui];
      const ReqInfo req = a.dv.reqs[unit.req];
      const int n_tiles = tiles_of(unit);
      const bool row_ok = row < unit.rows;
      const int pr = unit.row0 + (row_ok ? row : 0);
      const int t = pr / H;
      int limit = unit.kv_hi;
      if (a.g.causal) limit = min(limit, t + req.kv_len - req.qo_len + 1);
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n_tiles; ++j, ++g) {
        const int st = g & 1;
        mbar_wait(&sm.s_full[st], (g >> 1) & 1, wc);
        tc_fence_after();
        float sv[kN];
        tmem_ld32(lane_base + kSCol + st * kN, sv);
        tmem_ld32(lane_base + kSCol + st * kN + 32, sv + 32);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&sm.s_free[st]);
        const int kv0 = unit.kv_lo + j * kN;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < kN; ++c) {
          if (kv0 + c >= limit) sv[c] = -INFINITY;
          mx = fmaxf(mx, sv[c]);
        }
        const float m_cand = mx == -INFINITY ? -INFINITY : mx * scale;
        bool need = s_owner && m_cand > m + kRescaleThreshold;
        float alpha = need ? ex2(m - m_cand) : 1.f;
        // the high-half O row of lane 16 + i belongs to the S row of lane i
        const float alpha_o = __shfl_sync(0xffffffffu, alpha, lane & 15);
        const bool any = __any_sync(0xffffffffu, need);
        if (j > 0) {
          mbar_wait(&sm.o_done, (g - 1) & 1, wc);  // P buffer free, O stable
          tc_fence_after();
          if (any) {
            float ov[32];
#pragma unroll 1
            for (int c = 0; c < 256; c += 32) {
              tmem_ld32(lane_base + c, ov);
              tmem_ld_wait();
#pragma unroll
              for (int x = 0; x < 32; ++x) ov[x] *= alpha_o;
              tmem_st32(lane_base + c, ov);
            }
            tmem_st_wait();
          }
        }
        if (need) {
          l *= alpha;
          m = m_cand;
        }
        if (s_owner) {
          const float mu = m == -INFINITY ? 0.f : m;
          float rs = 0.f;
#pragma unroll
          for (int ch = 0; ch < kN / 8; ++ch) {
            float pv[8];
#pragma unroll
            for (int x = 0; x < 8; ++x) {
              pv[x] = ex2(fmaf(sv[ch * 8 + x], scale, -mu));
              rs += pv[x];
            }
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(p_addr + row * 128 + ((ch ^ (row & 7)) << 4)),
                         "r"(pack_bf16x2(pv[0], pv[1])), "r"(pack_bf16x2(pv[2], pv[3])),
                         "r"(pack_bf16x2(pv[4], pv[5])), "r"(pack_bf16x2(pv[6], pv[7]))
                         : "memory");
          }
          l += rs;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&sm.p_full);
      }
      // ------------------------------------------------------------ epilogue
      // (it also orders the next unit's first P store after this unit's last
      // P.V, which reads the same P buffer, and the O loads before the next
      // unit's first P.V overwrites O)
      if (n_tiles > 0) {
        mbar_wait(&sm.o_final, uq & 1, wc);
        tc_fence_after();
        ++uq;
      }
      const float l_row = __shfl_sync(0xffffffffu, l, lane & 15);
      const float m_row = __shfl_sync(0xffffffffu, m, lane & 15);
      const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
      const float lse2 = l_row > 0.f ? m_row + __log2f(l_row) : -INFINITY;
      const int half = s_owner ? 0 : 1;
      const size_t orow = (size_t)(req.q_start + t) * H + pr % H;
      for (int c = 0; c < 256; c += 32) {
        float ov[32];
        if (n_tiles > 0) {
          tmem_ld32(lane_base + c, ov);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) ov[x] = 0.f;
        }
        if (!row_ok) continue;
        const int d0 = half * 256 + c;
        if (unit.partial >= 0) {
          float* dst = a.dv.part_o + ((size_t)unit.partial * kRows + row) * kDc + d0;
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(dst + x) =
                make_float4(ov[x] * inv_l, ov[x + 1] * inv_l, ov[x + 2] * inv_l, ov[x + 3] * inv_l);
        } else {
          __nv_bfloat16* dst = a.o + orow * kDc + d0;
#pragma unroll
          for (int x = 0; x < 32; x += 8) {
            uint4 w;
            w.x = pack_bf16x2(ov[x + 0] * inv_l, ov[x + 1] * inv_l);
            w.y = pack_bf16x2(ov[x + 2] * inv_l, ov[x + 3] * inv_l);
            w.z = pack_bf16x2(ov[x + 4] * inv_l, ov[x + 5] * inv_l);
            w.w = pack_bf16x2(ov[x + 6] * inv_l, ov[x + 7] * inv_l);
            *reinterpret_cast<uint4*>(dst + x) = w;
          }
        }
      }
      if (row_ok && s_owner) {
        if (unit.partial >= 0) a.dv.part_lse[(size_t)unit.partial * kRows + row] = lse2;
        else if (a.lse) a.lse[orow] = lse2;
      }
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_mla(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices, const void* q_nope,
                       const void* q_pe, const void* ckv, const void* kpe, void* o, float* lse,
                       cudaStream_t stream) {
  if (g.num_units == 0 || g.num_ctas == 0) return cudaSuccess;
  Args a{static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(q_pe),
         static_cast<const __nv_bfloat16*>(ckv), static_cast<const __nv_bfloat16*>(kpe), kv_indices,
         static_cast<__nv_bfloat16*>(o), lse, g, dv};
  const size_t smem = sizeof(Smem) + 1024;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attrs_once((const void*)mla_kernel, (int)smem, configured, false);
  if (e != cudaSuccess) return e;
  mla_kernel<<<g.num_ctas, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace pkv
