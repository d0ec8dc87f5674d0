// Split-KV absorbed-MLA decode (one query token per request), built for HBM
// bandwidth.
//
// What it computes: the absorbed MLA attention of the MLA kernel (FlashInfer
// 0.2 release, "Fused MLA decode kernel"; definition
// mla_paged_prefill_causal_h16_ckv512_kpe64_ps1 in flashinfer-trace discussion
// #15) for qo_len = 1: every head of the token reads the same latent row per
// key, s_j = sm_scale (q_nope . ckv_j + q_pe . kpe_j), o = sum_j p_j ckv_j.
// One CTA handles one (request, KV chunk) and all its heads (up to 16, the
// M = 16 rows of mma.sync m16n8k16), so each latent byte is read from HBM
// once. Chunks of a split request write fp32 partial states that the merge
// kernel combines by their base-2 LSE ("Merge Attention States").
//
// At 30 flops per byte the path is HBM-bound. 4 warps stream 32-key tiles
// (32 KB of ckv + 4 KB of kpe) through a kStages-deep cp.async ring (about
// 100 KB or more in flight per SM, what HBM latency needs at full rate). Each warp computes S for 8 of the tile's keys over the full 576-wide
// key; the row maxima are exchanged through shared memory so that all warps
// use one running max, P goes to shared memory as bf16, and each warp
// accumulates O for its own 128 of the 512 latent columns over all 32 keys.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "launch_util.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = 4;
constexpr int kKeys = 32;    // keys per stage (8 per warp for S)
#ifndef PKV_MLA_DEC_STAGES
#define PKV_MLA_DEC_STAGES 2
#endif
constexpr int kStages = PKV_MLA_DEC_STAGES;  // ring depth: kStages - 1 tiles in flight
constexpr int kDc = 512;     // latent (ckv) width = value width
constexpr int kDr = 64;      // rope key (kpe) width
constexpr int kDq = kDc + kDr;
constexpr int kHeads = kDecodeRows;       // 16 MMA rows
constexpr int kQRow = kDq * 2;            // 1152 B
constexpr int kCkvRow = kDc * 2;          // 1024 B
constexpr int kKpeRow = kDr * 2;          // 128 B
constexpr int kQBytes = kHeads * kQRow;   // 18 KB
constexpr int kCkvBytes = kKeys * kCkvRow;
constexpr int kKpeBytes = kKeys * kKpeRow;
constexpr int kStageBytes = kCkvBytes + kKpeBytes;  // 36 KB
constexpr int kPRow = kKeys * 2;          // 64 B
constexpr int kPBytes = kHeads * kPRow;
constexpr int kOffQ = 0;
constexpr int kOffStage = kOffQ + kQBytes;
constexpr int kOffP = kOffStage + kStages * kStageBytes;
constexpr int kOffRed = kOffP + kPBytes;                 // [warps][16] floats
constexpr int kSmemBytes = kOffRed + kWarps * kHeads * 4;
static_assert(kOffStage % 128 == 0 && kOffP % 128 == 0 && kStageBytes % 128 == 0, "16-byte aligned tiles");
static_assert(kWarps * 128 == kDc, "each warp owns 128 latent columns of O");
static_assert(kWarps * 8 == kKeys, "each warp owns 8 keys of S");

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

// 16-byte chunk `c` of row `r` in a tile with `row_bytes` per row: the chunk's
// low three bits are XOR-ed with the row, so 8 consecutive rows at one logical
// chunk fall in 8 different bank groups (conflict-free ldmatrix). Row strides
// are multiples of 128 bytes.
__device__ __forceinline__ uint32_t sw_off(int r, int c, int row_bytes) {
  return (uint32_t)(r * row_bytes + (((c & ~7) | ((c ^ r) & 7)) << 4));
}
// P rows are 64 bytes (4 chunks): two rows share a 128-byte line, so the XOR
// uses row / 2.
__device__ __forceinline__ uint32_t p_off(int r, int c) { return (uint32_t)(r * kPRow + ((c ^ ((r >> 1) & 3)) << 4)); }

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

constexpr int kCtasPerSm = kSmemBytes <= 110 * 1024 ? 2 : 1;

__global__ void __launch_bounds__(kThreads, kCtasPerSm) mla_decode_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const WorkUnit unit = a.dv.units[blockIdx.x];
  const ReqInfo req = a.dv.reqs[unit.req];
  const int H = a.g.num_qo_heads, P = a.g.page_size, shift = a.g.page_shift;
  const int n = (unit.kv_hi - unit.kv_lo + kKeys - 1) / kKeys;
  const uint32_t sbase = smem_u32(smem);
  const uint32_t q_s = sbase + kOffQ, p_s = sbase + kOffP;
  float* red = reinterpret_cast<float*>(smem + kOffRed);

  // latent rows of tile j -> stage: 64 ckv chunks then 8 kpe chunks per key.
  // Four threads per key: one page-table read per thread, then 18 copies
  // (chunks q, q + 4, ...: each warp instruction covers 64 contiguous bytes of
  // 8 rows). The page id of a tile is read one tile ahead, during the previous
  // tile's math: read inside the copy loop it would serialise a global read
  // before every copy (the copies are ordered memory operations), and read
  // just before the loop it would stall the warp one memory latency a tile.
  static_assert(kThreads == 4 * kKeys, "four threads per key row");
  auto fetch_slot = [&](int j) -> long long {
    const int pos = unit.kv_lo + j * kKeys + (tid >> 2);
    if (pos >= unit.kv_hi) return -1;
    return (long long)__ldg(a.kv_indices + req.page0 + (pos >> shift)) * P + (pos & (P - 1));
  };
  auto load_tile = [&](int stage, long long slot_or_neg) {
    const uint32_t cdst = sbase + kOffStage + stage * kStageBytes;
    const uint32_t kdst = cdst + kCkvBytes;
    const int r = tid >> 2, q = tid & 3;
    const bool ok = slot_or_neg >= 0;
    const size_t slot = ok ? (size_t)slot_or_neg : 0;
    const __nv_bfloat16* csrc = a.ckv + slot * kDc;
    const __nv_bfloat16* ksrc = a.kpe + slot * kDr;
#pragma unroll
    for (int k = 0; k < kDq / 8 / 4; ++k) {
      const int ch = q + 4 * k;
      if (ch < kDc / 8) cp_async_16(cdst + sw_off(r, ch, kCkvRow), csrc + ch * 8, ok ? 16u : 0u);
      else cp_async_16(kdst + sw_off(r, ch - kDc / 8, kKpeRow), ksrc + (ch - kDc / 8) * 8, ok ? 16u : 0u);
    }
  };

  // Q: head h's [q_nope | q_pe] row, zero rows past the head count
  for (int c = tid; c < kHeads * (kDq / 8); c += kThreads) {
    const int h = c / (kDq / 8), ch = c % (kDq / 8);
    const bool ok = h < H;
    const size_t row = (size_t)req.q_start * H + (ok ? h : 0);
    const __nv_bfloat16* src = ch < kDc / 8 ? a.q_nope + row * kDc + ch * 8 : a.q_pe + row * kDr + (ch - kDc / 8) * 8;
    cp_async_16(q_s + sw_off(h, ch, kQRow), src, ok ? 16u : 0u);
  }
#pragma unroll
  for (int st = 0; st < kStages - 1; ++st) {
    if (st < n) load_tile(st, fetch_slot(st));
    cp_async_commit();  // group st (group 0 also holds Q)
  }
  long long slot_next = kStages - 1 < n ? fetch_slot(kStages - 1) : -1;  // tile j + kStages - 1

  const float scale = a.g.sm_scale_log2;
  const int r0 = lane >> 2;  // accumulator rows r0 and r0 + 8 (heads)
  float o_acc[16][4];        // this warp's 128 latent columns: 16 n-tiles of 8
#pragma unroll
  for (int i = 0; i < 16; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  for (int j = 0; j < n; ++j) {
    cp_async_wait<kStages - 2>();
    __syncthreads();  // tile j is in shared memory; every warp is done with tile j - 1
    if (j + kStages - 1 < n) load_tile((j + kStages - 1) % kStages, slot_next);
    cp_async_commit();
    if (j + kStages < n) slot_next = fetch_slot(j + kStages);
    const uint32_t cst = sbase + kOffStage + (j % kStages) * kStageBytes;
    const uint32_t kst = cst + kCkvBytes;

    // ---- S[16 x 8] for keys 8*warp .. 8*warp + 7 over the 576-wide key, in
    // four independent accumulators (a single one would chain all 36 MMAs)
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    {
      float sa[4][4] = {};
      const int qrow = (lane & 7) + ((lane >> 3) & 1) * 8;  // A: rows 0-15, chunk 2kk + lane / 16
      const int qhi = lane >> 4;
      const int krow = warp * 8 + (lane & 7);               // B: 4 matrices = chunks 2kk .. 2kk + 3
      const int kq = lane >> 3;
#pragma unroll
      for (int kk = 0; kk < kDq / 16; kk += 2) {
        uint32_t b0, b1, b2, b3;
        if (kk < kDc / 16) ldsm_x4(cst + sw_off(krow, 2 * kk + kq, kCkvRow), b0, b1, b2, b3);
        else ldsm_x4(kst + sw_off(krow, 2 * (kk - kDc / 16) + kq, kKpeRow), b0, b1, b2, b3);
        uint32_t qa[4], qb[4];
        ldsm_x4(q_s + sw_off(qrow, 2 * kk + qhi, kQRow), qa[0], qa[1], qa[2], qa[3]);
        ldsm_x4(q_s + sw_off(qrow, 2 * kk + 2 + qhi, kQRow), qb[0], qb[1], qb[2], qb[3]);
        mma16816(sa[(kk >> 1) & 1], qa, b0, b1);
        mma16816(sa[2 + ((kk >> 1) & 1)], qb, b2, b3);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) s[e] = (sa[0][e] + sa[1][e]) + (sa[2][e] + sa[3][e]);
    }
    // ---- scale, mask keys past the chunk, row max over this warp's 8 keys
    const int key0 = unit.kv_lo + j * kKeys + warp * 8 + (lane & 3) * 2;
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] = key0 + (e & 1) < unit.kv_hi ? s[e] * scale : -INFINITY;
    float mx0 = fmaxf(s[0], s[1]), mx1 = fmaxf(s[2], s[3]);
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    if ((lane & 3) == 0) {
      red[warp * kHeads + r0] = mx0;
      red[warp * kHeads + r0 + 8] = mx1;
    }
    __syncthreads();  // all warps' maxima are visible
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      mx0 = fmaxf(mx0, red[w * kHeads + r0]);
      mx1 = fmaxf(mx1, red[w * kHeads + r0 + 8]);
    }
    const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
    const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
    const float a0 = m0 == n0 ? 1.f : ex2(m0 - u0), a1 = m1 == n1 ? 1.f : ex2(m1 - u1);
    m0 = n0;
    m1 = n1;
    s[0] = ex2(s[0] - u0);
    s[1] = ex2(s[1] - u0);
    s[2] = ex2(s[2] - u1);
    s[3] = ex2(s[3] - u1);
    l0 = l0 * a0 + s[0] + s[1];
    l1 = l1 * a1 + s[2] + s[3];
    // P (bf16) for these 8 keys: chunk `warp` of rows r0 and r0 + 8
    {
      uint8_t* pb = smem + kOffP;
      *reinterpret_cast<uint32_t*>(pb + p_off(r0, warp) + (lane & 3) * 4) = pack_bf16x2(s[0], s[1]);
      *reinterpret_cast<uint32_t*>(pb + p_off(r0 + 8, warp) + (lane & 3) * 4) = pack_bf16x2(s[2], s[3]);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o_acc[i][0] *= a0;
      o_acc[i][1] *= a0;
      o_acc[i][2] *= a1;
      o_acc[i][3] *= a1;
    }
    __syncthreads();  // P of all 32 keys is visible
    // ---- O[:, 128 warp + (0..127)] += P[16 x 32] . ckv[32 keys x those columns]
    {
      const int prow = (lane & 7) + ((lane >> 3) & 1) * 8;
      const int phi = lane >> 4;
      const int mi = lane >> 3;
#pragma unroll
      for (int ks = 0; ks < kKeys / 16; ++ks) {
        uint32_t pa[4];
        ldsm_x4(p_s + p_off(prow, 2 * ks + phi), pa[0], pa[1], pa[2], pa[3]);
        const int vrow = ks * 16 + (lane & 7) + (mi & 1) * 8;
#pragma unroll
        for (int np = 0; np < 8; ++np) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(cst + sw_off(vrow, warp * 16 + np * 2 + (mi >> 1), kCkvRow), b0, b1, b2, b3);
          mma16816(o_acc[np * 2], pa, b0, b1);
          mma16816(o_acc[np * 2 + 1], pa, b2, b3);
        }
      }
    }
  }
  cp_async_wait<0>();

  // ---- row sums: each warp holds its keys' share; all warps used the same max
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
  __syncthreads();  // the last tile's maxima were read
  if ((lane & 3) == 0) {
    red[warp * kHeads + r0] = l0;
    red[warp * kHeads + r0 + 8] = l1;
  }
  __syncthreads();
  float L0 = 0.f, L1 = 0.f;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    L0 += red[w * kHeads + r0];
    L1 += red[w * kHeads + r0 + 8];
  }
  const float inv0 = L0 > 0.f ? 1.f / L0 : 0.f, inv1 = L1 > 0.f ? 1.f / L1 : 0.f;
  const float lse0 = L0 > 0.f ? m0 + __log2f(L0) : -INFINITY, lse1 = L1 > 0.f ? m1 + __log2f(L1) : -INFINITY;
  const int c0 = warp * 128 + (lane & 3) * 2;
  if (unit.partial >= 0) {
    const size_t base = (size_t)unit.partial * kDecodeRows;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (r0 < H)
        *reinterpret_cast<float2*>(a.dv.part_o + (base + r0) * kDc + c0 + i * 8) =
            make_float2(o_acc[i][0] * inv0, o_acc[i][1] * inv0);
      if (r0 + 8 < H)
        *reinterpret_cast<float2*>(a.dv.part_o + (base + r0 + 8) * kDc + c0 + i * 8) =
            make_float2(o_acc[i][2] * inv1, o_acc[i][3] * inv1);
    }
    if (warp == 0 && (lane & 3) == 0) {
      if (r0 < H) a.dv.part_lse[base + r0] = lse0;
      if (r0 + 8 < H) a.dv.part_lse[base + r0 + 8] = lse1;
    }
  } else {
    const size_t orow = (size_t)req.q_start * H;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (r0 < H)
        *reinterpret_cast<uint32_t*>(a.o + (orow + r0) * kDc + c0 + i * 8) = pack_bf16x2(o_acc[i][0] * inv0, o_acc[i][1] * inv0);
      if (r0 + 8 < H)
        *reinterpret_cast<uint32_t*>(a.o + (orow + r0 + 8) * kDc + c0 + i * 8) =
            pack_bf16x2(o_acc[i][2] * inv1, o_acc[i][3] * inv1);
    }
    if (warp == 0 && (lane & 3) == 0 && a.lse) {
      if (r0 < H) a.lse[orow + r0] = lse0;
      if (r0 + 8 < H) a.lse[orow + r0 + 8] = lse1;
    }
  }
}

}  // namespace

cudaError_t launch_mla_decode(const LaunchGeom& g, const DeviceView& dv, const int32_t* kv_indices,
                              const void* q_nope, const void* q_pe, const void* ckv, const void* kpe, void* o,
                              float* lse, cudaStream_t stream) {
  if (g.num_units == 0) return cudaSuccess;
  Args a{static_cast<const __nv_bfloat16*>(q_nope), static_cast<const __nv_bfloat16*>(q_pe),
         static_cast<const __nv_bfloat16*>(ckv), static_cast<const __nv_bfloat16*>(kpe), kv_indices,
         static_cast<__nv_bfloat16*>(o), lse, g, dv};
  // all of the unified L1 / shared array as shared memory, so two CTAs fit per SM
  static std::atomic<uint64_t> configured{0};
  cudaError_t e = set_smem_attrs_once((const void*)mla_decode_kernel, kSmemBytes, configured, true);
  if (e != cudaSuccess) return e;
  mla_decode_kernel<<<g.num_units, kThreads, kSmemBytes, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace pkv
