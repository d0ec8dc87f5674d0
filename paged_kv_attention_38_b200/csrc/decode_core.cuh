// Device-side body of the split-KV paged decode (one query token per request),
// shared by the planned decode kernel (decode_sm100.cu) and the decode entry
// point that allocates nothing (decode_noalloc.cu). Each caller decides which
// (request, kv head, KV range) a CTA takes and where its result goes; the
// attention over that range is this one function.
//
// What it computes: the paged attention of the prefill path with qo_len = 1
// (FlashInfer 0.7.4 documentation, flashinfer.decode; page table as in
// flashinfer-trace discussion #15, "Notes on fa3_gqa_prefill_v1"): the G query
// heads that share one kv head attend over keys [kv_lo, kv_hi) of the request,
// and the CTA writes either the final O / LSE rows or an fp32 partial state
// that a merge combines by its base-2 LSE ("Merge Attention States").
//
// The data path is HBM-bound (about 4 flops per byte at group 4), so it is
// shaped around bytes in flight: 4 warps stream 64-key tiles of K and V (32 KB
// per stage at head_dim 128) through a 3-stage cp.async ring, two CTAs per SM.
// The small contractions (group x 16 keys x head_dim) run on mma.sync m16n8k16
// only to keep the instruction count per byte low; the tensor core is not the
// bound. Query heads fill the M = 16 rows of the MMA, zero-padded past G.
#pragma once
#include <cuda_bf16.h>

#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {
namespace decode {

constexpr int kThreads = 128;
constexpr int kStages = 3;
constexpr int kTile = kDecodeTileN;  // keys per stage (16 per warp)

// Dynamic shared memory of one CTA: the K/V ring, reused by the final
// combination of the four warps' states.
template <int D>
constexpr size_t smem_bytes() {
  constexpr size_t pipe = (size_t)kStages * 2 * kTile * D * 2;
  constexpr size_t comb = (size_t)4 * 16 * D * 4 + 2 * 4 * 16 * 4;
  return pipe > comb ? pipe : comb;
}

// One CTA's job. The G query rows (and the G output rows) are consecutive
// rows of D elements.
struct Job {
  const __nv_bfloat16* q;       // [G][D] bf16
  const __nv_bfloat16* k;       // K pool (NHD [page][slot][Hk][D] or HND [page][Hk][slot][D])
  const __nv_bfloat16* v;       // V pool, same layout
  const int32_t* pages;         // the request's page ids (its slice of kv_indices)
  int kv_lo, kv_hi;             // keys of the request this CTA attends over
  int kv_head, G, Hk, P, shift; // kv head, group size (<= 16), kv heads, page size, log2(page size)
  float scale;                  // sm_scale * log2(e)
  float* part_o;                // non-null: write the fp32 partial state [G][D] here ...
  float* part_lse;              // ... and its base-2 LSE [G] here
  __nv_bfloat16* o;             // otherwise: bf16 O [G][D]
  float* lse;                   // and the LSE [G] (may be null)
};

// Byte offset of 16-byte chunk `ch` of key row `r` in a [kTile x D] tile with
// rows of D*2 bytes and the chunk index XOR-swizzled by row % 8 (conflict-free
// ldmatrix over 8 consecutive rows).
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

// kHnd: pages laid out [kv head][slot][D] (HND) instead of [slot][kv head][D].
// Every thread of the CTA (kThreads) calls this once; `smem` holds smem_bytes<D>().
template <int D, bool kHnd>
__device__ __forceinline__ void attend(uint8_t* smem, const Job& jb) {
  constexpr int kTileBytes = kTile * D * 2;
  constexpr int kChunks = D / 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = jb.G, Hk = jb.Hk, P = jb.P, shift = jb.shift;
  const int n = jb.kv_hi > jb.kv_lo ? (jb.kv_hi - jb.kv_lo + kTile - 1) / kTile : 0;
  const uint32_t sbase = smem_u32(smem);

  // Each warp reads only its own 16 key rows of every stage (rows 16 warp +
  // [0, 16)), so each warp also copies them itself and waits on its own copy
  // groups: no CTA-wide barrier per tile, the warps run at their own pace.
  // All page-table reads of a tile are issued before its copies: a read inside
  // the copy loop would wait for the previous copy to be issued (the copies
  // are ordered memory operations), serialising one global read per copy.
  constexpr int kPerLane = 16 * kChunks / 32;
  static_assert(16 * kChunks % 32 == 0, "whole copies per lane");
  // With pages of 16 keys or more, a warp's 16 rows (16-aligned positions) lie
  // in one page: one page id per lane, and the rows' offsets step by a constant.
  auto load_tile = [&](int j, int stage) {
    const uint32_t kdst = sbase + stage * 2 * kTileBytes;
    const uint32_t vdst = kdst + kTileBytes;
    if (P >= 16) {
      const int pos0 = jb.kv_lo + j * kTile + warp * 16;
      const int pg = pos0 < jb.kv_hi ? __ldg(jb.pages + (pos0 >> shift)) : -1;
      const size_t base = pg < 0 ? 0
                          : kHnd ? (((size_t)pg * Hk + jb.kv_head) * P + (pos0 & (P - 1))) * D
                                 : (((size_t)pg * P + (pos0 & (P - 1))) * Hk + jb.kv_head) * D;
      const size_t row_step = kHnd ? (size_t)D : (size_t)Hk * D;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) {
        const int c = lane + 32 * i;
        const int rr = c / kChunks, ch = c % kChunks;
        const bool ok = pg >= 0 && pos0 + rr < jb.kv_hi;
        const size_t off = ok ? base + rr * row_step + ch * 8 : 0;
        cp_async_16(kdst + kv_off<D>(warp * 16 + rr, ch), jb.k + off, ok ? 16u : 0u);
        cp_async_16(vdst + kv_off<D>(warp * 16 + rr, ch), jb.v + off, ok ? 16u : 0u);
      }
      return;
    }
    int page[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int pos = jb.kv_lo + j * kTile + warp * 16 + (lane + 32 * i) / kChunks;
      page[i] = pos < jb.kv_hi ? __ldg(jb.pages + (pos >> shift)) : -1;
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int c = lane + 32 * i;
      const int r = warp * 16 + c / kChunks, ch = c % kChunks;
      const int pos = jb.kv_lo + j * kTile + r;
      const bool ok = page[i] >= 0;
      size_t off = 0;
      if constexpr (kHnd)
        off = ok ? (((size_t)page[i] * Hk + jb.kv_head) * P + (pos & (P - 1))) * D + ch * 8 : 0;
      else
        off = ok ? (((size_t)page[i] * P + (pos & (P - 1))) * Hk + jb.kv_head) * D + ch * 8 : 0;
      cp_async_16(kdst + kv_off<D>(r, ch), jb.k + off, ok ? 16u : 0u);
      cp_async_16(vdst + kv_off<D>(r, ch), jb.v + off, ok ? 16u : 0u);
    }
  };

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < n) load_tile(s, s);
    cp_async_commit();
  }

  // Q as mma A fragments: rows = heads of the group (zero past G), k = head_dim.
  uint32_t qa[D / 16][4];
  {
    const int r0 = lane >> 2, kq = (lane & 3) * 2;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      auto ld = [&](int row, int col) -> uint32_t {
        if (row >= G) return 0u;
        return *reinterpret_cast<const uint32_t*>(jb.q + (size_t)row * D + col);
      };
      qa[kk][0] = ld(r0, kk * 16 + kq);
      qa[kk][1] = ld(r0 + 8, kk * 16 + kq);
      qa[kk][2] = ld(r0, kk * 16 + kq + 8);
      qa[kk][3] = ld(r0 + 8, kk * 16 + kq + 8);
    }
  }

  const float scale = jb.scale;
  float o_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows lane/4 and lane/4 + 8

  for (int j = 0; j < n; ++j) {
    cp_async_wait<kStages - 2>();
    __syncwarp();  // this warp's rows of tile j have landed; its reads of tile j - 1 are done
    if (j + kStages - 1 < n) load_tile(j + kStages - 1, (j + kStages - 1) % kStages);
    cp_async_commit();

    const uint32_t kst = sbase + (j % kStages) * 2 * kTileBytes;
    const uint32_t vst = kst + kTileBytes;
    // S[16 x 16] = Q . K^T for this warp's 16 keys
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
    // mask keys past the range's end, scale into the base-2 domain
    if (jb.kv_lo + (j + 1) * kTile <= jb.kv_hi) {  // the whole tile is in range (warp-uniform)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] *= scale;
    } else {
      const int key0 = jb.kv_lo + j * kTile + warp * 16 + (lane & 3) * 2;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + nt * 8 + (e & 1);
          s[nt][e] = key < jb.kv_hi ? s[nt][e] * scale : -INFINITY;
        }
      }
    }
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
    // O *= alpha only when some row of the warp moved its max (after the first
    // tiles the max rarely moves; the result is the same either way)
    if (__any_sync(0xffffffffu, a0 != 1.f || a1 != 1.f)) {
#pragma unroll
      for (int i = 0; i < D / 8; ++i) {
        o_acc[i][0] *= a0;
        o_acc[i][1] *= a0;
        o_acc[i][2] *= a1;
        o_acc[i][3] *= a1;
      }
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

  // ---- combine the 4 warps' states through shared memory
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* so = reinterpret_cast<float*>(smem);           // [4][16][D]
  float* sm_m = so + 4 * 16 * D;                         // [4][16]
  float* sm_l = sm_m + 4 * 16;                           // [4][16]
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
    if (jb.part_o) {
      jb.part_o[(size_t)row * D + d] = out;
      if (d == 0) jb.part_lse[row] = lse2;
    } else {
      jb.o[(size_t)row * D + d] = __float2bfloat16_rn(out);
      if (d == 0 && jb.lse) jb.lse[row] = lse2;
    }
  }
}

}  // namespace decode
}  // namespace pkv
