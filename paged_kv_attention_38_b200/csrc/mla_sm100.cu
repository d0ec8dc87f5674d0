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
// Two launches. mla_pack_kernel first copies every latent row a request's
// page table lists, ckv | kpe (1152 bytes), into a packed copy in the plan's
// workspace, request by request in key order. With page_size 1 the rows are
// scattered over the pool one by one, and a 16-byte-copy gather inside the
// attention kernel could not keep its tensor core fed; packed, each key tile
// is one dense [keys x 576] block that TMA moves in nine boxes. Every latent
// row is read by every query tile of its request, so the one pass over the
// pool (a few MB) is repaid many times; the packed copy stays in L2.
//
// mla_kernel then runs the attention. Shape choices for B200. A 128-row
// tile's 128 x 512 fp32 output alone would fill all 512 TMEM columns, and a
// 128 x 576 bf16 query tile (144 KB) leaves no room in shared memory for a key
// ring. So a CTA takes 64 packed (token, head) rows and runs M = 64 MMAs:
//   TMEM  O rows x latent[0,256)   lanes 16q + [0,16)  (q = sub-partition), cols [0,256)
//         O rows x latent[256,512) lanes 16q + [16,32),                     cols [0,256)
//         S (double buffer)        lanes 16q + [0,16),                      cols [256,288), [288,320)
//   (a 64-row accumulator uses half of each 32-lane sub-partition; the two
//   latent halves of O sit in the two halves, so a warp rescales both with one
//   32x32b load/store over columns [0,256) without touching S.)
//   SMEM  Q 64 x 576 (72 KB), a 4-stage TMA ring of 32-key latent tiles
//   (32 x 576, 36 KB: K and V at once, V being the ckv part of the same rows),
//   P 64 x 32 (in an 8 KB swizzled block).
// Both MMAs read their operands from shared memory, and two warps issue
// them: the S MMAs of the next tiles go in while the softmax and the P.V of
// the current one run, and with four stages three tiles are in flight behind
// the one being consumed. The kernel is persistent: one CTA per SM runs a
// host-planned list of units, its barrier phases running on across units.
// Warps: 0-3 softmax and epilogue (lanes 0-15 own S rows and the low O half,
// lanes 16-31 the high O half of the same rows), 4 TMEM allocator + S issuer,
// 5 TMA producer (one lane), 6 P.V issuer.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "launch_util.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"
#include "tma_util.h"

namespace pkv {

namespace {

constexpr int kRows = kMlaUnitRows;  // 64
constexpr int kN = kMlaTileN;        // keys per latent tile (32)
constexpr int kStages = 4;
constexpr int kDc = 512;
constexpr int kDr = 64;
constexpr int kDqk = kDc + kDr;      // 576
constexpr int kBlocks = kDqk / 64;   // 9 column blocks of 64 (128-byte rows)
constexpr int kQBlockBytes = kRows * 128;  // [64 rows x 64] bf16: 8 KB
constexpr int kKBlockBytes = kN * 128;     // [32 keys x 64] bf16: 4 KB
constexpr int kStageBytes = kBlocks * kKBlockBytes;
constexpr int kThreads = 224;
constexpr int kMmaWarp = 4;   // TMEM allocator + issuer of the S = Q K^T MMAs
constexpr int kProdWarp = 5;
constexpr int kPvWarp = 6;    // issuer of the O += P V MMAs
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSCol = 256;
constexpr float kRescaleThreshold = 8.0f;

struct __align__(1024) Smem {
  __nv_bfloat16 q[kBlocks * kRows * 64];
  __nv_bfloat16 kv[kStages][kBlocks * kN * 64];
  __nv_bfloat16 p[kRows * 64];  // P [64 rows x 32 keys] in the first 64 (logical) bytes of swizzled 128-byte rows
  uint64_t q_full;
  uint64_t q_empty;  // the unit's last QK^T MMAs are done: Q may be overwritten
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t s_free[2];
  uint64_t p_full;
  uint64_t o_done;
  uint64_t o_final;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) + 1024 <= 232448, "dynamic shared memory of one CTA (227 KB on sm_100)");

struct Args {
  CUtensorMap tm_q;    // q_nope as [total_q * H rows][512]
  CUtensorMap tm_qpe;  // q_pe as [total_q * H rows][64]
  CUtensorMap tm_lat;  // packed latent rows [packed_rows][576]
  __nv_bfloat16* o;
  float* lse;
  LaunchGeom g;
  DeviceView dv;
};

struct PackArgs {
  const __nv_bfloat16* ckv;
  const __nv_bfloat16* kpe;
  const int32_t* kv_indices;
  const ReqInfo* reqs;
  const int32_t* kv_row0;
  __nv_bfloat16* packed;
  int32_t batch, page_size, page_shift;
};

// Copy the latent rows of every request with queries into the packed copy:
// row kv_row0[b] + pos holds ckv (512) then kpe (64) of key pos of request b.
// A block covers 32 keys of one request (8 warps x 4 keys); a warp moves a
// 1152-byte row as 72 16-byte pieces, the loads of its four rows first.
constexpr int kPackKeys = 32;
__global__ void __launch_bounds__(256) mla_pack_kernel(const __grid_constant__ PackArgs a) {
  // the attention kernel may start now: it waits for this grid before its
  // first read of the packed rows (programmatic dependent launch)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int P = a.page_size, shift = a.page_shift;
  for (int b = blockIdx.y; b < a.batch; b += gridDim.y) {
    const ReqInfo req = a.reqs[b];
    if (req.qo_len == 0) continue;
    const int pos0 = blockIdx.x * kPackKeys + warp * 4;
    if (pos0 >= req.kv_len) continue;
    const int row0 = a.kv_row0[b];
    uint4 v[4][3];
    int n = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int pos = pos0 + i;
      if (pos < req.kv_len) {
        const size_t src = (size_t)__ldg(a.kv_indices + req.page0 + (pos >> shift)) * P + (pos & (P - 1));
        const uint4* c = reinterpret_cast<const uint4*>(a.ckv + src * kDc);
        v[i][0] = __ldg(c + lane);
        v[i][1] = __ldg(c + 32 + lane);
        if (lane < 8) v[i][2] = __ldg(reinterpret_cast<const uint4*>(a.kpe + src * kDr) + lane);
        n = i + 1;
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i < n) {
        uint4* d = reinterpret_cast<uint4*>(a.packed + (size_t)(row0 + pos0 + i) * kDqk);
        d[lane] = v[i][0];
        d[32 + lane] = v[i][1];
        if (lane < 8) d[64 + lane] = v[i][2];
      }
    }
  }
}

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
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
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

  if (warp == kProdWarp) {
    // ================================================================ producer (TMA, one lane)
    if (lane == 0) {
      tma_prefetch_desc(&a.tm_q);
      tma_prefetch_desc(&a.tm_qpe);
      tma_prefetch_desc(&a.tm_lat);
      int g = 0;   // latent tiles loaded by this CTA (stage g % kStages)
      int uq = 0;  // units with keys whose Q was loaded
      for (int ui = u_begin; ui < u_end; ++ui) {
        const WorkUnit unit = a.dv.units[ui];
        const int n_tiles = tiles_of(unit);
        if (n_tiles == 0) continue;
        const ReqInfo req = a.dv.reqs[unit.req];
        // Q, once the previous unit's QK^T MMAs have read the old one. The
        // unit's packed rows are consecutive rows of q viewed as [total_q * H]:
        // row (token t, head h) of the request is q_start * H + t * H + h.
        if (uq > 0) mbar_wait(&sm.q_empty, (uq - 1) & 1, wc);
        mbar_arrive_expect_tx(&sm.q_full, kBlocks * kQBlockBytes);
        const int qrow = req.q_start * H + unit.row0;
#pragma unroll
        for (int blk = 0; blk < kBlocks - 1; ++blk)
          tma_load_2d(smem_u32(sm.q) + blk * kQBlockBytes, &a.tm_q, &sm.q_full, blk * 64, qrow);
        tma_load_2d(smem_u32(sm.q) + (kBlocks - 1) * kQBlockBytes, &a.tm_qpe, &sm.q_full, 0, qrow);
        ++uq;
        // warm L2 with the next unit's Q so its load at the unit boundary is short
        if (ui + 1 < u_end) {
          const WorkUnit nu = a.dv.units[ui + 1];
          const int nrow = a.dv.reqs[nu.req].q_start * H + nu.row0;
#pragma unroll
          for (int blk = 0; blk < kBlocks - 1; ++blk) tma_prefetch_l2_2d(&a.tm_q, blk * 64, nrow);
          tma_prefetch_l2_2d(&a.tm_qpe, 0, nrow);
        }
        const int krow0 = a.dv.kv_row0[unit.req] + unit.kv_lo;
        if (g == 0) {
          // The kernel is launched as a programmatic dependent of the pack
          // kernel: everything above overlaps it, the packed rows are read only
          // after it has completed and its writes are visible.
          asm volatile("griddepcontrol.wait;" ::: "memory");
          asm volatile("fence.proxy.async.global;" ::: "memory");
        }
        for (int j = 0; j < n_tiles; ++j, ++g) {
          const int st = g % kStages;
          if (g >= kStages) mbar_wait(&sm.kv_empty[st], ((g / kStages) - 1) & 1, wc);
          mbar_arrive_expect_tx(&sm.kv_full[st], kStageBytes);
          const uint32_t dst = smem_u32(sm.kv[st]);
#pragma unroll
          for (int blk = 0; blk < kBlocks; ++blk)
            tma_load_2d(dst + blk * kKBlockBytes, &a.tm_lat, &sm.kv_full[st], blk * 64, krow0 + j * kN);
        }
      }
      // No TMA write may still land in this CTA's shared memory at exit: only
      // the last Q and the last kStages tiles can be in flight (every earlier
      // one was consumed before its buffer was refilled).
      if (uq > 0) mbar_drain(&sm.q_full, (uq - 1) & 1);
      for (int k = g - 1; k >= 0 && k >= g - kStages; --k) mbar_drain(&sm.kv_full[k % kStages], (k / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    // ================================================================ MMA issuers
    // Two warps issue the tensor-core work: warp kMmaWarp the S = Q K^T MMAs
    // (36 of N = 32 per tile, each cheap to run but about as costly to issue),
    // warp kPvWarp the O += P V MMAs. The two streams touch disjoint TMEM (S
    // buffers / O) and P sits in shared memory, so they need no mutual order;
    // each stream's own commits keep its barriers exact, and a tile's K/V
    // stage is released by the P.V commit, which implies its S finished (P
    // was computed from it). In each warp the whole warp runs the loop (waits,
    // descriptor arithmetic) and one elected lane issues each instruction.
    constexpr uint32_t idesc_s = idesc_bf16_f32(kRows, kN, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(kRows, 256, true);
    // Descriptors are built once; another stage, block or K-step only moves the
    // start address, the low 14-bit field (addr >> 4), so offsets are added in place.
    const uint64_t dq = sdesc_sw128(smem_u32(sm.q), 16, 1024);
    const uint64_t dp = sdesc_sw128(smem_u32(sm.p), 16, 1024);
    const uint64_t dk0 = sdesc_sw128(smem_u32(sm.kv[0]), 16, 1024);
    const uint64_t dv0 = sdesc_sw128(smem_u32(sm.kv[0]), kKBlockBytes, 1024);
    constexpr uint32_t kStageStep = (uint32_t)(kStageBytes >> 4);
    const bool s_issuer = warp == kMmaWarp;
    int g = 0;   // latent tiles of this CTA: stage g % kStages, S buffer g & 1 and the per-tile phases
    int uq = 0;  // units with keys: q_full / q_empty / o_final phases
    for (int ui = u_begin; ui < u_end; ++ui) {
      const int n_tiles = tiles_of(a.dv.units[ui]);
      if (n_tiles == 0) continue;
      if (s_issuer) {
        mbar_wait(&sm.q_full, uq & 1, wc);
        for (int j = 0; j < n_tiles; ++j, ++g) {
          const int st = g % kStages, sb = g & 1;
          mbar_wait(&sm.kv_full[st], (g / kStages) & 1, wc);
          if (g >= 2) mbar_wait(&sm.s_free[sb], ((g >> 1) - 1) & 1, wc);
          tc_fence_after();
          const uint64_t dk = dk0 + st * kStageStep;
#pragma unroll
          for (int b = 0; b < kBlocks; ++b) {  // four K-steps of one 64-column block per elect
            uint64_t da[4], db[4];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
              da[k4] = dq + ((b * kQBlockBytes + k4 * 32) >> 4);
              db[k4] = dk + ((b * kKBlockBytes + k4 * 32) >> 4);
            }
            umma4_bf16_ss_elect(tmem + kSCol + sb * kN, da, db, idesc_s, b > 0 ? 1u : 0u);
          }
          umma_commit_elect(&sm.s_full[sb]);
          if (j + 1 == n_tiles) umma_commit_elect(&sm.q_empty);  // the unit's last QK^T is issued
        }
      } else {
        // O += P V for each tile of the unit; the first tile overwrites O
        for (int j = 0; j < n_tiles; ++j, ++g) {
          const int st = g % kStages;
          mbar_wait(&sm.p_full, g & 1, wc);
          tc_fence_after();
#pragma unroll
          for (int nh = 0; nh < 2; ++nh) {
            const uint32_t d = tmem + (nh ? (16u << 16) : 0u);
#pragma unroll
            for (int kk = 0; kk < kN / 16; ++kk)
              umma_bf16_ss_elect(d, dp + ((kk * 32) >> 4),
                                 dv0 + st * kStageStep + ((4 * nh * kKBlockBytes + kk * 16 * 128) >> 4), idesc_o,
                                 (j > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit_elect(&sm.o_done);
          umma_commit_elect(&sm.kv_empty[st]);
        }
        umma_commit_elect(&sm.o_final);
      }
      ++uq;
    }
    // no MMA may still run when TMEM is released (the S stream's last
    // commits precede the last P.V, which needs every S of its unit)
    if (!s_issuer && uq > 0) mbar_drain(&sm.o_final, (uq - 1) & 1);
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
        const int sb = g & 1;
        mbar_wait(&sm.s_full[sb], (g >> 1) & 1, wc);
        tc_fence_after();
        float sv[kN];
        tmem_ld32(lane_base + kSCol + sb * kN, sv);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&sm.s_free[sb]);
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
            st_shared_v4(p_addr + row * 128 + ((ch ^ (row & 7)) << 4), pack_bf16x2(pv[0], pv[1]),
                         pack_bf16x2(pv[2], pv[3]), pack_bf16x2(pv[4], pv[5]), pack_bf16x2(pv[6], pv[7]));
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
      if (unit.partial >= 0) {
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
          float* dst = a.dv.part_o + ((size_t)unit.partial * kRows + row) * kDc + half * 256 + c;
#pragma unroll
          for (int x = 0; x < 32; x += 4)
            *reinterpret_cast<float4*>(dst + x) =
                make_float4(ov[x] * inv_l, ov[x + 1] * inv_l, ov[x + 2] * inv_l, ov[x + 3] * inv_l);
        }
      } else {
        // bf16 O, 64 columns of the thread's half-row at a time: 8 pieces of
        // 16 bytes. Each group of 8 lanes transposes its 8 half-rows x 8
        // pieces with xor butterflies, so that one store instruction writes
        // four whole 128-byte lines (lane 8g + i: piece i of half-row 8g + k)
        // instead of 32 pieces of 32 different lines.
        const int grp = lane & ~7, li = lane & 7;
        const size_t orow0 = (size_t)req.q_start * H + unit.row0;
        for (int c = 0; c < 256; c += 64) {
          float ov[64];
          if (n_tiles > 0) {
            tmem_ld32(lane_base + c, ov);
            tmem_ld32(lane_base + c + 32, ov + 32);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int x = 0; x < 64; ++x) ov[x] = 0.f;
          }
          uint4 pc[8];
#pragma unroll
          for (int k = 0; k < 8; ++k)
            pc[k] = make_uint4(pack_bf16x2(ov[8 * k + 0] * inv_l, ov[8 * k + 1] * inv_l),
                               pack_bf16x2(ov[8 * k + 2] * inv_l, ov[8 * k + 3] * inv_l),
                               pack_bf16x2(ov[8 * k + 4] * inv_l, ov[8 * k + 5] * inv_l),
                               pack_bf16x2(ov[8 * k + 6] * inv_l, ov[8 * k + 7] * inv_l));
#pragma unroll
          for (int sbit = 1; sbit < 8; sbit <<= 1) {
            const bool upper = (li & sbit) != 0;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              if (k & sbit) continue;
              uint4 snd = upper ? pc[k] : pc[k ^ sbit];
              uint4 rcv;
              rcv.x = __shfl_xor_sync(0xffffffffu, snd.x, sbit);
              rcv.y = __shfl_xor_sync(0xffffffffu, snd.y, sbit);
              rcv.z = __shfl_xor_sync(0xffffffffu, snd.z, sbit);
              rcv.w = __shfl_xor_sync(0xffffffffu, snd.w, sbit);
              if (upper) pc[k] = rcv;
              else pc[k ^ sbit] = rcv;
            }
          }
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int src = grp + k;               // lane whose half-row this store writes
            const int r = warp * 16 + (src & 15);  // its row of the unit
            if (r < unit.rows)
              *reinterpret_cast<uint4*>(a.o + (orow0 + r) * kDc + (src >> 4) * 256 + c + 8 * li) = pc[k];
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

std::atomic<uint64_t> g_configured{0};  // per-device shared-memory attribute of mla_kernel

}  // namespace

cudaError_t launch_mla(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices, const void* q_nope,
                       const void* q_pe, const void* ckv, const void* kpe, void* o, float* lse,
                       cudaStream_t stream) {
  if (g.num_units == 0 || g.num_ctas == 0) return cudaSuccess;
  // TMA row coordinates are int32
  const int64_t q_rows = (int64_t)g.total_q * g.num_qo_heads;
  if (q_rows <= 0 || q_rows > INT32_MAX) return cudaErrorInvalidValue;
  // 1. the packed latent rows of every request with queries
  if (g.packed_rows > 0) {
    PackArgs pa{static_cast<const __nv_bfloat16*>(ckv), static_cast<const __nv_bfloat16*>(kpe), kv_indices,
                dv.reqs, dv.kv_row0, static_cast<__nv_bfloat16*>(dv.packed), g.num_reqs, g.page_size,
                g.page_shift};
    const dim3 grid((unsigned)((g.max_kv_len + kPackKeys - 1) / kPackKeys), (unsigned)std::min(g.num_reqs, 65535));
    mla_pack_kernel<<<grid, 256, 0, stream>>>(pa);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 2. attention over the packed rows
  Args a{};
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.g = g;
  a.dv = dv;
  if (!make_map_2d(&a.tm_q, q_nope, kDc, q_rows, kDc * 2, 64, kRows) ||
      !make_map_2d(&a.tm_qpe, q_pe, kDr, q_rows, kDr * 2, 64, kRows) ||
      !make_map_2d(&a.tm_lat, dv.packed, kDqk, std::max(1, g.packed_rows), kDqk * 2, 64, kN))
    return cudaErrorInvalidValue;
  const size_t smem = sizeof(Smem) + 1024;
  cudaError_t e = set_smem_attrs_once((const void*)mla_kernel, (int)smem, g_configured, false);
  if (e != cudaSuccess) return e;
  // Programmatic dependent launch of the pack kernel: CTAs may start while it
  // runs (they read Q and the plan, both complete before it started, and wait
  // for it before the packed rows). Without a pack launch the previous kernel
  // on the stream is the caller's, so the launch is an ordinary one.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)g.num_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g.packed_rows > 0 ? 1 : 0;
  e = cudaLaunchKernelEx(&cfg, mla_kernel, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace pkv
