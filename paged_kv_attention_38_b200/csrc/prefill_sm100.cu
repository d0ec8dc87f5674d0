// Paged causal GQA prefill on sm_100a tensor cores (tcgen05, accumulators in TMEM).
//
// What it computes (flashinfer-trace discussion #15, definition
// gqa_paged_prefill_causal_h16_kv1_d128_ps64 and "Notes on fa3_gqa_prefill_v1";
// FlashInfer 0.2 release, "FlashAttention-3 template with block/vector
// sparsity"): for each work unit (request, kv head, 256 packed query rows,
// KV range), O = softmax(sm_scale Q K^T + causal mask) V over the keys the
// page table lists, plus the base-2 LSE of every row. K/V rows are gathered
// page by page through kv_indices: whole pages by TMA when page_size >= 8,
// single rows by 16-byte cp.async for page_size 1..4 (vector sparsity). The
// gather is the only difference from dense attention.
//
// CTA layout (384 threads, one work unit of two 128-row query tiles):
//   warps 0-3  softmax of query tile 0 (thread i owns row i = TMEM lane i)
//   warps 4-7  softmax of query tile 1
//   warp  8    TMEM allocator + MMA issuer (one lane)
//   warps 9-11 producer: TMA (one lane) or cp.async gather (96 threads)
// Shared memory: Q tiles (2 x 128 x D) and a 4-slot ring of 128 x D K or V
// tiles, all in 128-byte swizzled rows. TMEM (512 columns): S0 [0,128),
// S1 [128,256), O0 [256,384), O1 [384,512). After softmax reads S_i it writes
// P_i (bf16, two per column) over the first 64 columns of S_i, and the P.V
// MMA takes P_i straight from TMEM as its A operand.
//
// Per KV tile j the MMA warp issues, in order:
//   O0 += P0 V_j,  S0 = Q0 K_{j+1}^T,  O1 += P1 V_j,  S1 = Q1 K_{j+1}^T
// so the softmax of one query tile overlaps the MMAs of the other. The tensor
// core executes a CTA's MMAs in issue order, so S_i(j+1) overwrites P_i(j)
// only after O_i += P_i(j) V_j has read it, and the commit that signals S_i(j+1)
// also covers O_i += P_i(j) V_j: when softmax sees S_i(j+1), O_i is stable and
// may be rescaled in place.
//
// Online softmax runs in the base-2 domain (s' = s * sm_scale * log2 e,
// p = 2^(s' - m)). A row's running max m is only moved when the new tile's
// max exceeds it by more than 8 (p then stays below 2^8 in fp32 / bf16), so O
// is rescaled in TMEM a few times per row instead of once per tile.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "launch_util.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"
#include "tma_util.h"

namespace pkv {

namespace {

constexpr int kTileM = 128;
constexpr int kTiles = 2;
constexpr int kSlots = 4;
// Threads per CTA: 8 softmax warps, the MMA warp and the producer warps, 3 of
// them for the page-TMA instance (one lane issues TMA), 7 for the row-gather
// instance (its copy rate grows with the warps that issue 16-byte copies).
template <bool kRows>
constexpr int kThreadsOf = kRows ? 512 : 384;
constexpr int kMmaWarp = 8;
constexpr int kProdWarp0 = 9;
template <bool kRows>
constexpr int kProdThreadsOf = kThreadsOf<kRows> - kProdWarp0 * 32;
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;
template <bool kRows>
constexpr int kRegsSupportOf = kRows ? 56 : 96;
constexpr int kRegsSoftmax = 200;
// registers at launch: 65536 / threads, rounded down to a multiple of 8
static_assert(128 * kRegsSupportOf<false> + 256 * kRegsSoftmax <= 384 * 168, "register split exceeds the launch budget");
static_assert(256 * kRegsSupportOf<true> + 256 * kRegsSoftmax <= 512 * 128, "register split exceeds the launch budget");
static_assert(kTileM * kTiles == kPrefillUnitRows, "unit rows");

// Byte offset of 16-byte chunk `ch` of row `r` in a [128 x D] bf16 tile held as
// D/64 column blocks of [128 rows x 128 B], 128-byte swizzle (chunk ^ row % 8):
// the layout TMA SWIZZLE_128B writes and the UMMA SW128 descriptors read.
__device__ __forceinline__ uint32_t tile_off(int r, int ch) {
  return (uint32_t)((ch >> 3) * (kTileM * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4));
}

template <int D>
struct __align__(1024) Smem {
  __nv_bfloat16 q[kTiles][kTileM * D];
  __nv_bfloat16 kv[kSlots][kBlockN * D];
  alignas(128) uint8_t ostage[kPrefillUnitRows][128];  // epilogue staging (row gather instance): 128 B per row
  uint64_t q_full;
  uint64_t q_empty;  // the unit's last QK^T MMAs are done: Q may be overwritten
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t s_full[kTiles];
  uint64_t p_half[kTiles][2];  // P_i columns [0,64) / [64,128) written
  uint64_t o_final[kTiles];    // O_i of the unit is complete
  uint64_t mma_done;           // every MMA of the CTA is complete (exit)
  int32_t rowsrc[kBlockN];  // cp.async gather: pool row of each tile row, -1 = zero fill
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(offsetof(Smem<64>, ostage) % 128 == 0 && offsetof(Smem<128>, ostage) % 128 == 0,
              "16-byte shared stores into the staging rows");

struct Args {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int32_t* kv_indices;
  __nv_bfloat16* o;
  float* lse;
  LaunchGeom g;
  DeviceView dv;
  int32_t q_tma;      // Q tiles by TMA (group divides 128) or by cp.async
  int32_t kv_tma;     // K/V pages by TMA (page_size >= 8; the kRows = false instance) or by cp.async rows
  int32_t oob_row;    // a pool row index past the end: TMA zero-fills it
  // Per-kv-head scales of a quantised cache whose values were expanded to bf16
  // codes (NULL: 1), read by the kScaled instances only: K's multiplies the
  // scores, V's the output.
  const float* k_scale;
  const float* v_scale;
};

// kRows: K/V arrive as single rows by cp.async (page_size < 8) instead of whole
// pages by TMA. A template parameter, so each instance holds only its own
// producer code (the instances' register allocation is then independent).
//
// Persistent: CTA b runs work units [cta_ptr[b], cta_ptr[b + 1]) back to back.
// Barrier phases run on across units (counters of K/V items, KV tiles and
// units with keys), so the producer streams the next unit's Q and K/V and the
// tensor core starts its first QK^T while the softmax warps still write the
// previous unit's output.
template <int D, bool kRows, bool kHnd, bool kScaled>
__global__ void __launch_bounds__(kThreadsOf<kRows>, 1) prefill_kernel(const __grid_constant__ Args a) {
  constexpr int kProdThreads = kProdThreadsOf<kRows>;
  constexpr int kRegsSupport = kRegsSupportOf<kRows>;
  extern __shared__ uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const int u_begin = a.dv.cta_ptr[blockIdx.x];
  const int u_end = a.dv.cta_ptr[blockIdx.x + 1];
  const int G = a.g.group;
  auto tiles_of = [](const WorkUnit& u) { return (u.kv_hi - u.kv_lo + kBlockN - 1) / kBlockN; };

  if (tid == 0) {
    mbar_init(&sm.q_full, a.q_tma ? 1 : kProdThreads);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], kRows ? kProdThreads : 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int i = 0; i < kTiles; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.p_half[i][0], kTileM);
      mbar_init(&sm.p_half[i][1], kTileM);
      mbar_init(&sm.o_final[i], 1);
    }
    mbar_init(&sm.mma_done, 1);
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
  // Registers: 384 threads x 168 at launch = 64512 (page instance) or 512 x 128
  // = 65536 (row gather). The MMA/producer warpgroups (warps 8 and up) drop to
  // kRegsSupport, the two softmax warpgroups rise to kRegsSoftmax: 128 x 96 +
  // 256 x 200 = 63488 <= 64512, 256 x 56 + 256 x 200 = 65536. Each role's code
  // sits under its own setmaxnreg so the compiler allocates it with that budget.
  if (warp >= kMmaWarp) {
    setmaxnreg_dec<kRegsSupport>();
  if (warp >= kProdWarp0) {
    // ================================================================ producer
    const int pt = tid - kProdWarp0 * 32;
    constexpr int kChunks = D / 8;
    const int P = a.g.page_size, shift = a.g.page_shift, Hk = a.g.num_kv_heads;
    if (pt == 0) {
      if (a.q_tma) tma_prefetch_desc(&a.tm_q);
      if constexpr (!kRows) {
        tma_prefetch_desc(&a.tm_k);
        tma_prefetch_desc(&a.tm_v);
      }
    }
    // Q tile i of a unit by TMA: rows of 128 / G tokens x G heads from this token on.
    auto q_token = [&](const WorkUnit& u, const ReqInfo& rq, int i) { return rq.q_start + (u.row0 + i * kTileM) / G; };
    int kc = 0;  // K/V items issued (item 2j is K_j, 2j+1 is V_j; slot = item % kSlots)
    int uq = 0;  // units with keys whose Q was loaded
    for (int ui = u_begin; ui < u_end; ++ui) {
      const WorkUnit unit = a.dv.units[ui];
      const int n_tiles = tiles_of(unit);
      if (n_tiles == 0) continue;  // the CTA only writes zeros for it
      const ReqInfo req = a.dv.reqs[unit.req];
      // ---- Q tiles, once the previous unit's QK^T MMAs have read the old ones
      if (uq > 0) mbar_wait(&sm.q_empty, (uq - 1) & 1, wc);
      if (a.q_tma) {
        if (pt == 0) {
          mbar_arrive_expect_tx(&sm.q_full, kTiles * kTileM * D * 2);
          for (int i = 0; i < kTiles; ++i) {
            const int tok = q_token(unit, req, i);
#pragma unroll
            for (int h = 0; h < D / 64; ++h)
              tma_load_3d(smem_u32(sm.q[i]) + h * (kTileM * 128), &a.tm_q, &sm.q_full, h * 64, unit.kv_head * G, tok);
          }
          // warm L2 with the next unit's Q so its load at the unit boundary is short
          if (ui + 1 < u_end) {
            const WorkUnit nu = a.dv.units[ui + 1];
            const ReqInfo nr = a.dv.reqs[nu.req];
            for (int i = 0; i < kTiles; ++i)
#pragma unroll
              for (int h = 0; h < D / 64; ++h)
                tma_prefetch_l2_3d(&a.tm_q, h * 64, nu.kv_head * G, q_token(nu, nr, i));
          }
        }
      } else {
        const size_t head_stride = (size_t)a.g.num_qo_heads * D;
        for (int c = pt; c < kTiles * kTileM * kChunks; c += kProdThreads) {
          const int r = c / kChunks, ch = c % kChunks;
          const bool ok = r < unit.rows;
          const __nv_bfloat16* src = a.q;
          if (ok) {
            const int pr = unit.row0 + r;
            src = a.q + (size_t)(req.q_start + pr / G) * head_stride + (size_t)(unit.kv_head * G + pr % G) * D + ch * 8;
          }
          cp_async_16(smem_u32(sm.q[r / kTileM]) + tile_off(r % kTileM, ch), src, ok ? 16u : 0u);
        }
        cp_async_arrive_noinc(&sm.q_full);
      }
      ++uq;
      // ---- K / V items
      const int n_pages_req = (req.kv_len + P - 1) >> shift;
      for (int k = 0; k < 2 * n_tiles; ++k, ++kc) {
        const int slot = kc & (kSlots - 1);
        const int j = k >> 1;
        const bool is_v = k & 1;
        const int pos0 = unit.kv_lo + j * kBlockN;
        if constexpr (!kRows) {
          if (pt == 0) {
            if (kc >= kSlots) mbar_wait(&sm.empty[slot], ((kc >> 2) - 1) & 1, wc);
            mbar_arrive_expect_tx(&sm.full[slot], kBlockN * D * 2);
            const CUtensorMap* tm = is_v ? &a.tm_v : &a.tm_k;
            const uint32_t dst = smem_u32(sm.kv[slot]);
            if constexpr (kHnd) {
              // HND view [page x kv head][slot][D]: one kv head's slots of a page are contiguous
              if (P >= kBlockN) {
                const int ph = __ldg(a.kv_indices + req.page0 + (pos0 >> shift)) * Hk + unit.kv_head;
#pragma unroll
                for (int h = 0; h < D / 64; ++h)
                  tma_load_3d(dst + h * (kTileM * 128), tm, &sm.full[slot], h * 64, pos0 & (P - 1), ph);
              } else {
                const int npc = kBlockN >> shift;
                const int lp0 = pos0 >> shift;
                for (int pi = 0; pi < npc; ++pi) {
                  const int lp = lp0 + pi;
                  const int ph = lp < n_pages_req ? __ldg(a.kv_indices + req.page0 + lp) * Hk + unit.kv_head : a.oob_row;
#pragma unroll
                  for (int h = 0; h < D / 64; ++h)
                    tma_load_3d(dst + h * (kTileM * 128) + pi * P * 128, tm, &sm.full[slot], h * 64, 0, ph);
                }
              }
            } else {
            if (P >= kBlockN) {
              const int page = __ldg(a.kv_indices + req.page0 + (pos0 >> shift));
              const int row = page * P + (pos0 & (P - 1));
#pragma unroll
              for (int h = 0; h < D / 64; ++h) tma_load_3d(dst + h * (kTileM * 128), tm, &sm.full[slot], h * 64, unit.kv_head, row);
            } else {
              const int npc = kBlockN >> shift;
              const int lp0 = pos0 >> shift;
              for (int pi = 0; pi < npc; ++pi) {
                const int lp = lp0 + pi;
                const int row = lp < n_pages_req ? __ldg(a.kv_indices + req.page0 + lp) * P : a.oob_row;
#pragma unroll
                for (int h = 0; h < D / 64; ++h)
                  tma_load_3d(dst + h * (kTileM * 128) + pi * P * 128, tm, &sm.full[slot], h * 64, unit.kv_head, row);
              }
            }
            }
          }
        } else {
          if (kc >= kSlots) mbar_wait(&sm.empty[slot], ((kc >> 2) - 1) & 1, wc);
          if (!is_v) {
            named_bar_sync(1, kProdThreads);  // the previous tile's copies have all been issued
            for (int r = pt; r < kBlockN; r += kProdThreads) {
              const int pos = pos0 + r;
              int src = -1;
              if (pos < unit.kv_hi) src = __ldg(a.kv_indices + req.page0 + (pos >> shift)) * P + (pos & (P - 1));
              sm.rowsrc[r] = src;
            }
            named_bar_sync(1, kProdThreads);
          }
          {
            // thread pt copies 16-byte column ch of rows r0, r0 + kRowStep, ...:
            // the source row is read once per row and the column offset is fixed.
            const __nv_bfloat16* base = (is_v ? a.v : a.k) + unit.kv_head * D;
            const uint32_t dst = smem_u32(sm.kv[slot]);
            constexpr int kRowStep = kProdThreads / kChunks;
            const int ch = pt % kChunks;
            const uint32_t col_off = (uint32_t)((ch >> 3) * (kTileM * 128) + ((ch & 7) << 4));
            const size_t row_stride = (size_t)Hk * D;
            for (int r = pt / kChunks; r < kBlockN; r += kRowStep) {
              const int src = sm.rowsrc[r];
              const __nv_bfloat16* g = a.k;
              if constexpr (kHnd) {  // page src / P, slot src % P, [page][kv head][slot][D]
                if (src >= 0)
                  g = (is_v ? a.v : a.k) + (((size_t)(src >> shift) * Hk + unit.kv_head) * P + (src & (P - 1))) * D + ch * 8;
              } else {
                if (src >= 0) g = base + (size_t)src * row_stride + ch * 8;
              }
              cp_async_16(dst + r * 128 + (col_off ^ ((r & 7) << 4)), g, src >= 0 ? 16u : 0u);
            }
          }
          cp_async_arrive_noinc(&sm.full[slot]);
        }
      }
    }
    cp_async_wait<0>();
    // Make sure no TMA write into this CTA's shared memory is still in flight at
    // exit: only the last kSlots items and the last Q can be (every earlier one
    // was consumed before its slot was refilled).
    if (pt == 0) {
      if (a.q_tma && uq > 0) mbar_drain(&sm.q_full, (uq - 1) & 1);
      if constexpr (!kRows)
        for (int k = kc - 1; k >= 0 && k >= kc - kSlots; --k) mbar_drain(&sm.full[k & (kSlots - 1)], (k >> 2) & 1);
    }
  } else if (warp == kMmaWarp) {
    // ================================================================ MMA issuer
    // The whole warp runs this loop (waits, descriptor arithmetic) so its
    // operands stay in uniform registers; one elected lane issues each
    // tcgen05.mma / commit. (Run from a single divergent lane, the same loop
    // cost about twice the instructions per MMA and left the tensor core idle.)
    constexpr uint32_t idesc_s = idesc_bf16_f32(kTileM, kBlockN, false);
    constexpr uint32_t idesc_o = idesc_bf16_f32(kTileM, D, true);
    auto wait_item = [&](int k) {
      mbar_wait(&sm.full[k & (kSlots - 1)], (k >> 2) & 1, wc);
      fence_proxy_async_smem();  // cp.async rows were written through the generic proxy
      tc_fence_after();
    };
    // Descriptors are built once; a K-step or another buffer only moves the
    // start address, the low 14-bit field (addr >> 4), so offsets are added in place.
    const uint64_t dq0 = sdesc_sw128(smem_u32(sm.q[0]), 16, 1024);
    const uint64_t dk0 = sdesc_sw128(smem_u32(sm.kv[0]), 16, 1024);
    const uint64_t dv0 = sdesc_sw128(smem_u32(sm.kv[0]), kBlockN * 128, 1024);
    constexpr uint32_t kQStep = (kTileM * D * 2) >> 4;      // one Q tile
    constexpr uint32_t kSlotStep = (kBlockN * D * 2) >> 4;  // one K/V slot
    // S_i = Q_i K^T for the K item `item`
    auto issue_s = [&](int i, int item) {
      const uint64_t bq = dq0 + i * kQStep, bk = dk0 + (item & (kSlots - 1)) * kSlotStep;
#pragma unroll
      for (int k0 = 0; k0 < D / 16; k0 += 4) {  // the four K-steps of a 64-column block per elect
        uint64_t da[4], db[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const uint32_t off = (((k0 + x) >> 2) * (kTileM * 128) + ((k0 + x) & 3) * 32) >> 4;
          da[x] = bq + off;
          db[x] = bk + off;
        }
        umma4_bf16_ss_elect(tmem + i * kBlockN, da, db, idesc_s, k0 > 0 ? 1u : 0u);
      }
      umma_commit_elect(&sm.s_full[i]);
    };
    // O_i += P_i V for kv columns [64h, 64h + 64) of the V item `item`: K-steps 4h..4h+3.
    // `first`: the unit's first KV tile, which overwrites O_i.
    auto issue_pv_half = [&](int i, int item, int h, bool first) {
      const uint64_t bv = dv0 + (item & (kSlots - 1)) * kSlotStep;
      uint32_t ta[4];
      uint64_t db[4];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int kk = 4 * h + x;
        ta[x] = tmem + i * kBlockN + kk * 8;
        db[x] = bv + ((kk * 16 * 128) >> 4);
      }
      umma4_bf16_ts_elect(tmem + 256 + i * 128, ta, db, idesc_o, (!first || h > 0) ? 1u : 0u);
    };
    int jt = 0;  // KV tiles done by this CTA (all units): s_full / p_half phases
    int uq = 0;  // units with keys: q_full / q_empty / o_final phases
    for (int ui = u_begin; ui < u_end; ++ui) {
      const int n_tiles = tiles_of(a.dv.units[ui]);
      if (n_tiles == 0) continue;
      mbar_wait(&sm.q_full, uq & 1, wc);
      fence_proxy_async_smem();
      wait_item(2 * jt);
      issue_s(0, 2 * jt);
      issue_s(1, 2 * jt);
      umma_commit_elect(&sm.empty[(2 * jt) & (kSlots - 1)]);
      if (n_tiles == 1) umma_commit_elect(&sm.q_empty);
      for (int j = 0; j < n_tiles; ++j) {
        const int jj = jt + j;  // this CTA's KV tile count: item 2jj is K, 2jj+1 is V
        const bool more = j + 1 < n_tiles;
        mbar_wait(&sm.p_half[0][0], jj & 1, wc);
        wait_item(2 * jj + 1);
        issue_pv_half(0, 2 * jj + 1, 0, j == 0);
        mbar_wait(&sm.p_half[0][1], jj & 1, wc);
        tc_fence_after();
        issue_pv_half(0, 2 * jj + 1, 1, j == 0);
        if (more) {
          wait_item(2 * jj + 2);
          issue_s(0, 2 * jj + 2);
        } else {
          umma_commit_elect(&sm.o_final[0]);
        }
        mbar_wait(&sm.p_half[1][0], jj & 1, wc);
        tc_fence_after();
        issue_pv_half(1, 2 * jj + 1, 0, j == 0);
        mbar_wait(&sm.p_half[1][1], jj & 1, wc);
        tc_fence_after();
        issue_pv_half(1, 2 * jj + 1, 1, j == 0);
        umma_commit_elect(&sm.empty[(2 * jj + 1) & (kSlots - 1)]);
        if (more) {
          issue_s(1, 2 * jj + 2);
          umma_commit_elect(&sm.empty[(2 * jj + 2) & (kSlots - 1)]);
          if (j + 2 == n_tiles) umma_commit_elect(&sm.q_empty);
        } else {
          umma_commit_elect(&sm.o_final[1]);
        }
      }
      jt += n_tiles;
      ++uq;
    }
    // no MMA may still run when TMEM is released
    umma_commit_elect(&sm.mma_done);
    mbar_drain(&sm.mma_done, 0);
    __syncwarp();
  }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ================================================================ softmax
    const int ti = warp >> 2;          // query tile
    const int r = tid & (kTileM - 1);  // row in tile == TMEM lane
    const int ru = ti * kTileM + r;    // row in unit
    const float scale0 = a.g.sm_scale_log2;
    const uint32_t lane_base = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const uint32_t s_tm = lane_base + ti * kBlockN;
    const uint32_t o_tm = lane_base + 256 + ti * 128;
    int jt = 0, uq = 0;
    for (int ui = u_begin; ui < u_end; ++ui) {
      // Only what the KV loop needs stays live across it; the epilogue reads
      // the unit again (the softmax warps run close to their register budget).
      int n_tiles, kv_lo, limit;
      float scale = scale0;  // base-2 score scale (times this unit's kv-head K scale)
      {
        const WorkUnit unit = a.dv.units[ui];
        const ReqInfo req = a.dv.reqs[unit.req];
        if constexpr (kScaled) {
          if (a.k_scale) scale *= a.k_scale[unit.kv_head];
        }
        n_tiles = tiles_of(unit);
        kv_lo = unit.kv_lo;
        const int t = (unit.row0 + (ru < unit.rows ? ru : 0)) / G;
        limit = unit.kv_hi;
        if (a.g.causal) limit = min(limit, t + req.kv_len - req.qo_len + 1);
      }
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n_tiles; ++j) {
        mbar_wait(&sm.s_full[ti], (jt + j) & 1, wc);
        tc_fence_after();
        float sv[kBlockN];
        tmem_ld64(s_tm, sv);
        tmem_ld64(s_tm + 64, sv + 64);
        tmem_ld_wait();
        const int kv0 = kv_lo + j * kBlockN;
        const bool whole = kv0 + kBlockN <= limit;
        if (!whole) {
#pragma unroll
          for (int c = 0; c < kBlockN; ++c)
            if (kv0 + c >= limit) sv[c] = -INFINITY;
        }
        // row max: four independent 3-input max chains
        float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < kBlockN; c += 8) {
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], sv[c], sv[c + 1]);
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], sv[c + 2], sv[c + 3]);
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], sv[c + 4], sv[c + 5]);
          mx4[(c >> 3) & 3] = fmax3(mx4[(c >> 3) & 3], sv[c + 6], sv[c + 7]);
        }
        const float mx = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]);
        const float m_cand = mx == -INFINITY ? -INFINITY : mx * scale;
        const bool need = m_cand > m + kRescaleThreshold;
        const float alpha = need ? ex2(m - m_cand) : 1.f;
        const bool rescale_o = j > 0 && __any_sync(0xffffffffu, need);
        if (need) {
          l *= alpha;
          m = m_cand;
        }
        const float mu = m == -INFINITY ? 0.f : m;
        // p = 2^(s * scale - m) (masked columns hold -inf and give 0), packed to
        // bf16 and stored over S in 32-column chunks; each half of P is published
        // as soon as it is in TMEM so the P.V MMAs can start on it.
        const float2 scale2 = make_float2(scale, scale);
        const float2 nmu2 = make_float2(-mu, -mu);
        float2 rs2a = make_float2(0.f, 0.f), rs2b = make_float2(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t pw[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = h * 64 + 2 * e;
            const float2 x = ffma2(make_float2(sv[c], sv[c + 1]), scale2, nmu2);
            float2 pp;
            pp.x = ex2(x.x);
            pp.y = ex2(x.y);
            if (e & 1) rs2b = fadd2(rs2b, pp);
            else rs2a = fadd2(rs2a, pp);
            pw[e] = pack_bf16x2(pp.x, pp.y);
          }
          tmem_st32(s_tm + h * 32, reinterpret_cast<const float*>(pw));
          // O_i *= alpha before the first P.V MMA of this tile adds to it (the
          // S commit covered the previous tile's P.V). Done here, with half of
          // S already consumed, so the rescale's registers fit beside the rest.
          if (h == 0 && rescale_o) {
            float ov[32];
#pragma unroll
            for (int c = 0; c < D; c += 32) {
              tmem_ld32(o_tm + c, ov);
              tmem_ld_wait();
#pragma unroll
              for (int x = 0; x < 32; ++x) ov[x] *= alpha;
              tmem_st32(o_tm + c, ov);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&sm.p_half[ti][h]);
        }
        l += (rs2a.x + rs2a.y) + (rs2b.x + rs2b.y);
      }
      // ---------------------------------------------------------- epilogue
      // (the loads of O_i complete before this thread's next P arrive, so the
      // next unit's first P.V MMA cannot overwrite O_i under them)
      if (n_tiles > 0) {
        mbar_wait(&sm.o_final[ti], uq & 1, wc);
        tc_fence_after();
      }
      const WorkUnit unit = a.dv.units[ui];
      const ReqInfo req = a.dv.reqs[unit.req];
      const bool row_ok = ru < unit.rows;
      const int pr = unit.row0 + (row_ok ? ru : 0);
      float inv_l = l > 0.f ? 1.f / l : 0.f;
      if constexpr (kScaled) {
        if (a.v_scale) inv_l *= a.v_scale[unit.kv_head];
      }
      const float lse2 = l > 0.f ? m + __log2f(l) : -INFINITY;
      const int tok = req.q_start + pr / G;
      const int h = unit.kv_head * G + pr % G;
      if constexpr (kRows) {
        // Rows leave through this warp's staging tile in shared memory, 128 bytes
        // of each of its 32 rows per pass, so that every global store
        // instruction writes four whole 128-byte lines (eight lanes per row)
        // instead of a 16-byte piece of 32 different lines. fp32 partial state
        // (split units) takes 32 columns per pass, bf16 O 64.
        const bool part = unit.partial >= 0;
        char* my_dst = nullptr;
        if (row_ok)
          my_dst = part ? reinterpret_cast<char*>(a.dv.part_o + ((size_t)unit.partial * kPrefillUnitRows + ru) * D)
                        : reinterpret_cast<char*>(a.o + ((size_t)tok * a.g.num_qo_heads + h) * D);
        // this warp's 32 rows are ru & ~31 ... (ru & ~31) + 31; this thread's is lane ru & 31
        const int rl = ru & 31;
        const uint32_t stage = smem_u32(sm.ostage[ru & ~31]);
        const int n_pass = part ? D / 32 : D / 64;
        const uint32_t my_row = stage + rl * 128;
        for (int ps = 0; ps < n_pass; ++ps) {
          // this row's 128 bytes of the pass -> 8 swizzled 16-byte chunks
          if (part) {
            float ov[32];
            if (n_tiles > 0) {
              tmem_ld32(o_tm + ps * 32, ov);
              tmem_ld_wait();
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              uint32_t w[4];
#pragma unroll
              for (int x = 0; x < 4; ++x) w[x] = __float_as_uint(n_tiles > 0 ? ov[4 * k + x] * inv_l : 0.f);
              st_shared_v4(my_row + ((k ^ (rl & 7)) << 4), w[0], w[1], w[2], w[3]);
            }
          } else {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              float ov[32];
              if (n_tiles > 0) {
                tmem_ld32(o_tm + ps * 64 + q * 32, ov);
                tmem_ld_wait();
              }
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                uint32_t w[4];
#pragma unroll
                for (int x = 0; x < 4; ++x)
                  w[x] = n_tiles > 0 ? pack_bf16x2(ov[8 * k + 2 * x] * inv_l, ov[8 * k + 2 * x + 1] * inv_l) : 0u;
                st_shared_v4(my_row + (((4 * q + k) ^ (rl & 7)) << 4), w[0], w[1], w[2], w[3]);
              }
            }
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int rr = 4 * it + (rl >> 3), k = rl & 7;
            char* d = reinterpret_cast<char*>(__shfl_sync(0xffffffffu, reinterpret_cast<uintptr_t>(my_dst), rr));
            const uint4 v = ld_shared_v4(stage + rr * 128 + ((k ^ (rr & 7)) << 4));
            if (d) *reinterpret_cast<uint4*>(d + ps * 128 + k * 16) = v;
          }
          __syncwarp();
        }
        if (row_ok) {
          if (part) a.dv.part_lse[(size_t)unit.partial * kPrefillUnitRows + ru] = lse2;
          else if (a.lse) a.lse[(size_t)tok * a.g.num_qo_heads + h] = lse2;
        }
      } else {
        if (unit.partial >= 0) {
          float* dst = a.dv.part_o + ((size_t)unit.partial * kPrefillUnitRows + ru) * D;
#pragma unroll
          for (int c = 0; c < D; c += 32) {
            float ov[32];
            if (n_tiles > 0) {
              tmem_ld32(o_tm + c, ov);
              tmem_ld_wait();
            } else {
#pragma unroll
              for (int x = 0; x < 32; ++x) ov[x] = 0.f;
            }
            if (row_ok) {
#pragma unroll
              for (int x = 0; x < 32; x += 4)
                *reinterpret_cast<float4*>(dst + c + x) =
                    make_float4(ov[x] * inv_l, ov[x + 1] * inv_l, ov[x + 2] * inv_l, ov[x + 3] * inv_l);
            }
          }
          if (row_ok) a.dv.part_lse[(size_t)unit.partial * kPrefillUnitRows + ru] = lse2;
        } else {
          // 64 columns of the row at a time (8 pieces of 16 bytes). Each group
          // of 8 lanes (8 consecutive rows) transposes its 8 rows x 8 pieces
          // with xor butterflies, so that one store instruction writes four
          // 128-byte runs (lane 8g + i: piece i of row 8g + k) instead of 32
          // pieces of 32 different lines. A row's address comes from its lane.
          char* my_dst = row_ok ? reinterpret_cast<char*>(a.o + ((size_t)tok * a.g.num_qo_heads + h) * D) : nullptr;
          const int li = lane & 7, grp = lane & ~7;
#pragma unroll
          for (int c = 0; c < D; c += 64) {
            float ov[64];
            if (n_tiles > 0) {
              tmem_ld32(o_tm + c, ov);
              tmem_ld32(o_tm + c + 32, ov + 32);
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
                const uint4 snd = upper ? pc[k] : pc[k ^ sbit];
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
              char* d = reinterpret_cast<char*>(
                  __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(my_dst), grp + k));
              if (d) *reinterpret_cast<uint4*>(d + c * 2 + li * 16) = pc[k];
            }
          }
          if (row_ok && a.lse) a.lse[(size_t)tok * a.g.num_qo_heads + h] = lse2;
        }
      }
      tc_fence_before();
      jt += n_tiles;
      if (n_tiles > 0) ++uq;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

// 3-D bf16 tensor [rows][heads][D] (D contiguous), box {64, box_heads, box_rows},
// 128-byte swizzle, zero fill out of bounds.
bool make_map(CUtensorMap* m, const void* base, int D, int heads, int64_t rows, int box_heads, int box_rows) {
  auto fn = tensor_map_encoder();
  if (!fn || rows <= 0) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)heads, (cuuint64_t)rows};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)heads * D * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D, bool kRows, bool kHnd, bool kScaled = false>
cudaError_t launch_as(const Args& a, cudaStream_t stream) {
  const size_t smem = sizeof(Smem<D>) + 1024;
  static std::atomic<uint64_t> configured{0};
  cudaError_t e =
      set_smem_attrs_once((const void*)prefill_kernel<D, kRows, kHnd, kScaled>, (int)smem, configured, false);
  if (e != cudaSuccess) return e;
  prefill_kernel<D, kRows, kHnd, kScaled><<<a.g.num_ctas, kThreadsOf<kRows>, smem, stream>>>(a);
  return cudaGetLastError();
}

// One instance per K/V path and page layout, so that each holds only its own
// address arithmetic (the NHD instances are unchanged by the HND ones), and
// NHD instances with per-kv-head scales for the expanded FP8 cache (the bf16
// instances carry none of that code).
template <int D>
cudaError_t launch(const Args& a, cudaStream_t stream) {
  if (a.k_scale || a.v_scale) {
    if (a.g.kv_layout == 1) return cudaErrorInvalidValue;
    return a.kv_tma ? launch_as<D, false, false, true>(a, stream) : launch_as<D, true, false, true>(a, stream);
  }
  if (a.g.kv_layout == 1)
    return a.kv_tma ? launch_as<D, false, true>(a, stream) : launch_as<D, true, true>(a, stream);
  return a.kv_tma ? launch_as<D, false, false>(a, stream) : launch_as<D, true, false>(a, stream);
}

}  // namespace

cudaError_t launch_prefill(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices, const void* q,
                           const void* k, const void* v, int32_t num_pages, void* o, float* lse,
                           const float* k_scale, const float* v_scale, cudaStream_t stream) {
  if (g.num_units == 0 || g.num_ctas == 0) return cudaSuccess;
  Args a{};
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k = static_cast<const __nv_bfloat16*>(k);
  a.v = static_cast<const __nv_bfloat16*>(v);
  a.kv_indices = kv_indices;
  a.o = static_cast<__nv_bfloat16*>(o);
  a.lse = lse;
  a.g = g;
  a.dv = dv;
  const int64_t pool_rows = (int64_t)num_pages * g.page_size;
  const bool hnd = g.kv_layout == 1;
  // K/V tensor-map rows: NHD pool rows (slots), HND (page, kv head) pairs
  const int64_t map_rows = hnd ? (int64_t)num_pages * g.num_kv_heads : pool_rows;
  a.oob_row = (int32_t)std::min<int64_t>(map_rows, INT32_MAX);
  a.q_tma = (kTileM % g.group == 0) &&
            make_map(&a.tm_q, q, g.head_dim, g.num_qo_heads, g.total_q, g.group, kTileM / g.group);
  const int box = g.page_size < kBlockN ? g.page_size : kBlockN;
  if (hnd)  // [page x kv head][slot][D]: dims {D, page_size, pages x heads}, box {64, slots, 1}
    a.kv_tma = g.page_size >= 8 && map_rows < INT32_MAX &&
               make_map(&a.tm_k, k, g.head_dim, g.page_size, map_rows, box, 1) &&
               make_map(&a.tm_v, v, g.head_dim, g.page_size, map_rows, box, 1);
  else
    a.kv_tma = g.page_size >= 8 && pool_rows < INT32_MAX &&
               make_map(&a.tm_k, k, g.head_dim, g.num_kv_heads, pool_rows, 1, box) &&
               make_map(&a.tm_v, v, g.head_dim, g.num_kv_heads, pool_rows, 1, box);
  if (g.head_dim == 128) return launch<128>(a, stream);
  if (g.head_dim == 64) return launch<64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pkv
