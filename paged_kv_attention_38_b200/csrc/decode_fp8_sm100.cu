// Split-KV paged decode over a per-head-scale FP8 KV cache.
//
// What it computes: the paged decode of the bf16 kernel (FlashInfer 0.7.4
// documentation, flashinfer.decode) with K and V pools of FP8 E4M3 codes and
// one fp32 scale per kv head for K and for V ("[Roadmap] FlashInfer v0.2 to
// v0.3", milestone "Per Head Scale Quantized KV-Cache"): the cache's value is
// decode(code) * scale[kv head]. The K scale is folded into the score scale
// and the V scale into the output, so the kernel only has to turn codes into
// numbers the tensor cores take.
//
// The data path is the bf16 decode's at half the bytes per key: one CTA per
// (request, kv head, KV chunk), 4 warps, 64-key tiles of K and V codes
// (16 KB per stage at head_dim 128) through a 4-stage cp.async ring, three
// CTAs per SM. Each warp owns 16 keys of a tile and builds its mma.sync
// m16n8k16 operand fragments straight from the codes in shared memory (one
// cvt.rn.f16x2.e4m3x2 per pair of codes; every E4M3 value is exact in f16),
// so every code byte crosses the shared-memory port once. Two permutations
// make each thread's codes contiguous:
//   - S = Q K^T sums over the head dimension in any order, so Q and K share
//     one permutation of it: in k-step kk, lane (g, c) = (lane / 4, lane % 4)
//     takes the four dims c * D/4 + 4 kk + [0, 4), i.e. the D/4 contiguous
//     codes [c * D/4, (c + 1) * D/4) of its key row cover all its k-steps.
//   - In O += P V, column n of n-tile nt stands for dim (D/8) n + nt, so lane
//     (g, c) reads the D/8 contiguous codes [(D/8) g, (D/8)(g + 1)) of each of
//     its four key rows; the combine at the end writes each accumulator to
//     its dim.
// Q is scaled once per CTA by a power of two that brings its largest |q| to
// [2^13, 2^14) before the f16 rounding (undone exactly in the score scale), so
// any finite bf16 query stays in range. P is in [0, 1]; accumulators are fp32.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "launch_util.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

namespace {

constexpr int kThreads = 128;
constexpr int kStages = 4;
constexpr int kTile = kDecodeTileN;  // keys per stage (16 per warp)

struct Args {
  const __nv_bfloat16* q;
  const uint8_t* k;  // E4M3 codes, NHD pages
  const uint8_t* v;
  const float* k_scale;  // [num_kv_heads], or null for 1
  const float* v_scale;
  const int32_t* kv_indices;
  __nv_bfloat16* o;
  float* lse;
  LaunchGeom g;
  DeviceView dv;
};

// Byte offset of 16-byte chunk `ch` of key row `r` in a [kTile x D] code tile.
// D = 128: eight chunks per row, XOR-swizzled by row % 8, so that the K reads
// (eight rows, four chunks) and the V reads (four rows, eight chunks) of a
// quarter warp hit distinct banks. D = 64: rows of four chunks, unswizzled.
template <int D>
__device__ __forceinline__ uint32_t code_off(int r, int ch) {
  if constexpr (D == 128) return (uint32_t)(r * D + ((ch ^ (r & 7)) << 4));
  return (uint32_t)(r * D + (ch << 4));
}

__device__ __forceinline__ void mma16816_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Four E4M3 codes (bytes 0..3 of w) -> two f16x2: lo = (byte 0, byte 1),
// hi = (byte 2, byte 3).
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\t"
      "mov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// `n` bytes (16 or 8) of shared memory into words w[0..n/4).
template <int N>
__device__ __forceinline__ void ld_codes(uint32_t addr, uint32_t* w) {
  if constexpr (N == 16) {
    const uint4 v = ld_shared_v4(addr);
    w[0] = v.x, w[1] = v.y, w[2] = v.z, w[3] = v.w;
  } else if constexpr (N == 32) {
    const uint4 v0 = ld_shared_v4(addr), v1 = ld_shared_v4(addr + 16);
    w[0] = v0.x, w[1] = v0.y, w[2] = v0.z, w[3] = v0.w;
    w[4] = v1.x, w[5] = v1.y, w[6] = v1.z, w[7] = v1.w;
  } else {
    asm volatile("ld.shared.v2.b32 {%0, %1}, [%2];" : "=r"(w[0]), "=r"(w[1]) : "r"(addr) : "memory");
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 3) decode_fp8_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kCodeTile = kTile * D;  // bytes of one K (or V) code tile
  constexpr int kChunks = D / 16;       // 16-byte chunks of codes per key row
  constexpr int kKSteps = D / 16;       // k-steps of S = Q K^T
  constexpr int kNTiles = D / 8;        // n-tiles of O += P V
  constexpr int kKBytes = D / 4;        // contiguous K codes of a lane per key row
  constexpr int kVBytes = D / 8;        // contiguous V codes of a lane per key row
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lg = lane >> 2, lc = lane & 3;
  const WorkUnit unit = a.dv.units[blockIdx.x];
  const ReqInfo req = a.dv.reqs[unit.req];
  const int G = a.g.group, Hk = a.g.num_kv_heads, P = a.g.page_size, shift = a.g.page_shift;
  const int n = (unit.kv_hi - unit.kv_lo + kTile - 1) / kTile;
  const uint32_t sbase = smem_u32(smem);

  // Each warp reads only its own 16 key rows of every stage (rows 16 warp +
  // [0, 16)), so each warp also copies them itself and waits on its own copy
  // groups: no CTA-wide barrier per tile, the warps run at their own pace.
  // Page ids are read one tile ahead of the copies that use them, during the
  // previous tile's math, so no warp waits a global-memory latency per tile.
  constexpr int kPerLane = 16 * kChunks / 32;
  static_assert(16 * kChunks % 32 == 0, "whole copies per lane");
  // With pages of 16 keys or more, a warp's 16 rows (16-aligned positions) lie
  // in one page: one page id per lane, and the rows' offsets step by Hk * D.
  const bool one_page = P >= 16;
  auto fetch_pages = [&](int j, int* page) {
    if (one_page) {
      const int pos = unit.kv_lo + j * kTile + warp * 16;
      page[0] = pos < unit.kv_hi ? __ldg(a.kv_indices + req.page0 + (pos >> shift)) : -1;
      return;
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int pos = unit.kv_lo + j * kTile + warp * 16 + (lane + 32 * i) / kChunks;
      page[i] = pos < unit.kv_hi ? __ldg(a.kv_indices + req.page0 + (pos >> shift)) : -1;
    }
  };
  auto load_tile = [&](int j, int stage, const int* page) {
    const uint32_t kdst = sbase + stage * 2 * kCodeTile;
    const uint32_t vdst = kdst + kCodeTile;
    if (one_page) {
      const int pos0 = unit.kv_lo + j * kTile + warp * 16;
      const size_t base =
          page[0] >= 0 ? (((size_t)page[0] * P + (pos0 & (P - 1))) * Hk + unit.kv_head) * D : 0;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) {
        const int c = lane + 32 * i;
        const int rr = c / kChunks, ch = c % kChunks;
        const bool ok = page[0] >= 0 && pos0 + rr < unit.kv_hi;
        const size_t off = ok ? base + (size_t)rr * Hk * D + ch * 16 : 0;
        cp_async_16(kdst + code_off<D>(warp * 16 + rr, ch), a.k + off, ok ? 16u : 0u);
        cp_async_16(vdst + code_off<D>(warp * 16 + rr, ch), a.v + off, ok ? 16u : 0u);
      }
      return;
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int c = lane + 32 * i;
      const int r = warp * 16 + c / kChunks, ch = c % kChunks;
      const int pos = unit.kv_lo + j * kTile + r;
      const bool ok = page[i] >= 0;
      const size_t off = ok ? (((size_t)page[i] * P + (pos & (P - 1))) * Hk + unit.kv_head) * D + ch * 16 : 0;
      cp_async_16(kdst + code_off<D>(r, ch), a.k + off, ok ? 16u : 0u);
      cp_async_16(vdst + code_off<D>(r, ch), a.v + off, ok ? 16u : 0u);
    }
  };

  int page_next[kPerLane];  // ids of tile (j + kStages - 1), read during tile j - 1
#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < n) {
      fetch_pages(s, page_next);
      load_tile(s, s, page_next);
    }
    cp_async_commit();
  }
  if (kStages - 1 < n) fetch_pages(kStages - 1, page_next);

  // Q as f16 mma A fragments in the permuted head-dim order: rows = heads of
  // the group (zero past G); in k-step kk this lane holds dims
  // lc * D/4 + 4 kk + [0, 2) (a0, a1) and + [2, 4) (a2, a3).
  uint32_t qa[kKSteps][4];
  float qscale = 1.f;
  {
    const __nv_bfloat16* qrow = a.q + ((size_t)req.q_start * a.g.num_qo_heads + unit.kv_head * G) * D;
    float qf[kKSteps][8];
    float qmax = 0.f;
#pragma unroll
    for (int kk = 0; kk < kKSteps; ++kk) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = lg + 8 * h;
        float4 f = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row < G) {
          const uint2 raw = *reinterpret_cast<const uint2*>(qrow + (size_t)row * D + lc * kKBytes + 4 * kk);
          const float2 f01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
          const float2 f23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
          f = make_float4(f01.x, f01.y, f23.x, f23.y);
        }
        qf[kk][4 * h + 0] = f.x, qf[kk][4 * h + 1] = f.y, qf[kk][4 * h + 2] = f.z, qf[kk][4 * h + 3] = f.w;
        qmax = fmaxf(qmax, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) qmax = fmaxf(qmax, __shfl_xor_sync(0xffffffffu, qmax, o));
    // power of two bringing qmax to [2^13, 2^14): exact in fp32, undone in the score scale
    if (qmax > 0.f && qmax < INFINITY) {
      const int e = (int)((__float_as_uint(qmax) >> 23) & 0xFF) - 127;  // floor(log2 qmax), normal qmax
      const int se = min(13 - max(e, -126), 127);
      qscale = __uint_as_float((uint32_t)(127 + se) << 23);
    }
#pragma unroll
    for (int kk = 0; kk < kKSteps; ++kk) {
      qa[kk][0] = pack_f16x2(qf[kk][0] * qscale, qf[kk][1] * qscale);  // row lg,     dims +0, +1
      qa[kk][1] = pack_f16x2(qf[kk][4] * qscale, qf[kk][5] * qscale);  // row lg + 8, dims +0, +1
      qa[kk][2] = pack_f16x2(qf[kk][2] * qscale, qf[kk][3] * qscale);  // row lg,     dims +2, +3
      qa[kk][3] = pack_f16x2(qf[kk][6] * qscale, qf[kk][7] * qscale);  // row lg + 8, dims +2, +3
    }
  }

  const float ks = a.k_scale ? a.k_scale[unit.kv_head] : 1.f;
  const float vs = a.v_scale ? a.v_scale[unit.kv_head] : 1.f;
  const float scale = a.g.sm_scale_log2 * ks / qscale;
  float o_acc[kNTiles][4];
#pragma unroll
  for (int i = 0; i < kNTiles; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows lg and lg + 8

  for (int j = 0; j < n; ++j) {
    cp_async_wait<kStages - 2>();
    __syncwarp();  // this warp's rows of tile j have landed; its reads of tile j - 1 are done
    if (j + kStages - 1 < n) load_tile(j + kStages - 1, (j + kStages - 1) % kStages, page_next);
    cp_async_commit();
    if (j + kStages < n) fetch_pages(j + kStages, page_next);

    const uint32_t kst = sbase + (j % kStages) * 2 * kCodeTile;
    const uint32_t vst = kst + kCodeTile;
    const int r0 = warp * 16;  // this warp's 16 keys of the tile
    // S[16 x 16] = Q . K^T: n-tile t holds keys r0 + 8t + [0, 8); this lane's
    // B fragments come from key r0 + 8t + lg, codes [lc * D/4, +D/4)
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int r = r0 + 8 * t + lg;
      uint32_t w[kKBytes / 4];
      if constexpr (D == 128) {
        ld_codes<16>(kst + code_off<D>(r, 2 * lc), w);
        ld_codes<16>(kst + code_off<D>(r, 2 * lc + 1), w + 4);
      } else {
        ld_codes<16>(kst + code_off<D>(r, lc), w);
      }
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
        uint32_t b0, b1;
        e4m3x4_to_f16x2x2(w[kk], b0, b1);
        mma16816_f16(s[t], qa[kk], b0, b1);
      }
    }
    // mask keys past the unit's end, scale into the base-2 domain
    if (unit.kv_lo + (j + 1) * kTile <= unit.kv_hi) {  // the whole tile is in range (warp-uniform)
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] *= scale;
    } else {
      const int key0 = unit.kv_lo + j * kTile + r0 + lc * 2;
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + nt * 8 + (e & 1);
          s[nt][e] = key < unit.kv_hi ? s[nt][e] * scale : -INFINITY;
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
      for (int i = 0; i < kNTiles; ++i) {
        o_acc[i][0] *= a0;
        o_acc[i][1] *= a0;
        o_acc[i][2] *= a1;
        o_acc[i][3] *= a1;
      }
    }
    // P as the A fragment: keys r0 + 2lc, +1 (a0, a1) and r0 + 8 + 2lc, +1 (a2, a3)
    uint32_t pa[4];
    pa[0] = pack_f16x2(s[0][0], s[0][1]);
    pa[1] = pack_f16x2(s[0][2], s[0][3]);
    pa[2] = pack_f16x2(s[1][0], s[1][1]);
    pa[3] = pack_f16x2(s[1][2], s[1][3]);
    // O += P V: the B fragment of n-tile nt pairs the codes of keys (2lc, 2lc + 1)
    // and (2lc + 8, 2lc + 9) at dim (D/8) lg + nt, byte nt of this lane's run
    {
      uint32_t va[kVBytes / 4], vb[kVBytes / 4], vc[kVBytes / 4], vd[kVBytes / 4];
      const int rk = r0 + 2 * lc;
      if constexpr (D == 128) {
        ld_codes<16>(vst + code_off<D>(rk, lg), va);
        ld_codes<16>(vst + code_off<D>(rk + 1, lg), vb);
        ld_codes<16>(vst + code_off<D>(rk + 8, lg), vc);
        ld_codes<16>(vst + code_off<D>(rk + 9, lg), vd);
      } else {
        ld_codes<8>(vst + rk * D + lg * kVBytes, va);
        ld_codes<8>(vst + (rk + 1) * D + lg * kVBytes, vb);
        ld_codes<8>(vst + (rk + 8) * D + lg * kVBytes, vc);
        ld_codes<8>(vst + (rk + 9) * D + lg * kVBytes, vd);
      }
#pragma unroll
      for (int wi = 0; wi < kVBytes / 4; ++wi) {
        uint32_t b01[4], b89[4];
        e4m3x4_to_f16x2x2(__byte_perm(va[wi], vb[wi], 0x5140), b01[0], b01[1]);
        e4m3x4_to_f16x2x2(__byte_perm(va[wi], vb[wi], 0x7362), b01[2], b01[3]);
        e4m3x4_to_f16x2x2(__byte_perm(vc[wi], vd[wi], 0x5140), b89[0], b89[1]);
        e4m3x4_to_f16x2x2(__byte_perm(vc[wi], vd[wi], 0x7362), b89[2], b89[3]);
#pragma unroll
        for (int x = 0; x < 4; ++x) mma16816_f16(o_acc[4 * wi + x], pa, b01[x], b89[x]);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // ---- combine the 4 warps' states through shared memory; accumulator
  // (nt, column 2lc + x) of this lane is dim (D/8)(2lc + x) + nt
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  float* so = reinterpret_cast<float*>(smem);           // [4][16][D]
  float* sm_m = so + 4 * 16 * D;                         // [4][16]
  float* sm_l = sm_m + 4 * 16;                           // [4][16]
  {
    float* ow = so + warp * 16 * D;
#pragma unroll
    for (int nt = 0; nt < kNTiles; ++nt) {
      const int d0 = kVBytes * (2 * lc) + nt, d1 = kVBytes * (2 * lc + 1) + nt;
      ow[lg * D + d0] = o_acc[nt][0];
      ow[lg * D + d1] = o_acc[nt][1];
      ow[(lg + 8) * D + d0] = o_acc[nt][2];
      ow[(lg + 8) * D + d1] = o_acc[nt][3];
    }
    if (lc == 0) {
      sm_m[warp * 16 + lg] = m0;
      sm_m[warp * 16 + lg + 8] = m1;
      sm_l[warp * 16 + lg] = l0;
      sm_l[warp * 16 + lg + 8] = l1;
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
    const float out = L > 0.f ? acc / L * vs : 0.f;
    const float lse2 = L > 0.f ? mu + __log2f(L) : -INFINITY;
    if (unit.partial >= 0) {
      const size_t prow = (size_t)unit.partial * kDecodeRows + row;
      a.dv.part_o[prow * D + d] = out;
      if (d == 0) a.dv.part_lse[prow] = lse2;
    } else {
      const size_t orow = (size_t)req.q_start * a.g.num_qo_heads + unit.kv_head * G + row;
      a.o[orow * D + d] = __float2bfloat16_rn(out);
      if (d == 0 && a.lse) a.lse[orow] = lse2;
    }
  }
}

template <int D>
cudaError_t launch(const Args& a, cudaStream_t stream) {
  const size_t pipe = (size_t)kStages * 2 * kTile * D;
  const size_t comb = (size_t)4 * 16 * D * 4 + 2 * 4 * 16 * 4;
  const size_t smem = pipe > comb ? pipe : comb;
  auto kern = decode_fp8_kernel<D>;
  // all of the unified L1 / shared array as shared memory, so three CTAs fit per SM
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attrs_once((const void*)kern, (int)smem, configured, true);
  if (e != cudaSuccess) return e;
  kern<<<a.g.num_units, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_fp8(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices, const void* q,
                              const void* k, const void* v, const float* k_scale, const float* v_scale, void* o,
                              float* lse, cudaStream_t stream) {
  if (g.num_units == 0) return cudaSuccess;
  Args a{static_cast<const __nv_bfloat16*>(q), static_cast<const uint8_t*>(k), static_cast<const uint8_t*>(v),
         k_scale, v_scale, kv_indices, static_cast<__nv_bfloat16*>(o), lse, g, dv};
  if (g.head_dim == 128) return launch<128>(a, stream);
  if (g.head_dim == 64) return launch<64>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace pkv
