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
// The data path is the bf16 decode's, at half the bytes per key: 4 warps
// stream 64-key tiles of K and V codes (16 KB per stage at head_dim 128)
// through a 3-stage cp.async ring. Each warp converts its own 16 keys of the
// tile to f16 (every E4M3 value is exact in f16, one cvt.rn.f16x2.e4m3x2 per
// pair) into the swizzled rows of one f16 working tile, first K for
// S = Q K^T, then V into the same rows for O += P V, so only warp barriers
// separate conversion and use and 64 KB of shared memory lets three CTAs
// share an SM (the conversion makes the kernel latency-bound with two). Both
// products run on mma.sync m16n8k16 with f16 operands (Q is rounded to f16
// once, P is in [0, 1]) and fp32 accumulators; query heads fill the M = 16
// rows.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "launch_util.h"
#include "pkv_internal.h"
#include "sm100_ptx.cuh"

namespace pkv {

namespace {

constexpr int kThreads = 128;
constexpr int kStages = 3;
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

// Byte offset of 16-byte chunk `ch` (8 f16) of key row `r` in a [kTile x D]
// f16 tile, chunk index XOR-swizzled by row % 8 (conflict-free ldmatrix).
template <int D>
__device__ __forceinline__ uint32_t f16_off(int r, int ch) {
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

__device__ __forceinline__ void mma16816_f16(float* d, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Two E4M3 codes (low byte = lower element) -> f16x2 (low half = lower element).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t out;
  const unsigned short in = (unsigned short)two_codes;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(out) : "h"(in));
  return out;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D>
__global__ void __launch_bounds__(kThreads, 3) decode_fp8_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int kCodeTile = kTile * D;       // bytes of one K (or V) code tile
  constexpr int kChunks = D / 16;            // 16-byte chunks of codes per key row
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const WorkUnit unit = a.dv.units[blockIdx.x];
  const ReqInfo req = a.dv.reqs[unit.req];
  const int G = a.g.group, Hk = a.g.num_kv_heads, P = a.g.page_size, shift = a.g.page_shift;
  const int n = (unit.kv_hi - unit.kv_lo + kTile - 1) / kTile;
  const uint32_t sbase = smem_u32(smem);
  // One f16 working tile: each warp converts its 16 K rows, computes S, then
  // converts its 16 V rows into the same rows for P.V.
  const uint32_t f16t = sbase + kStages * 2 * kCodeTile;

  // All page-table reads of a tile are issued before its copies.
  constexpr int kPerThread = kTile * kChunks / kThreads;
  static_assert(kTile * kChunks % kThreads == 0, "whole copies per thread");
  auto load_tile = [&](int j, int stage) {
    const uint32_t kdst = sbase + stage * 2 * kCodeTile;
    const uint32_t vdst = kdst + kCodeTile;
    int page[kPerThread];
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const int pos = unit.kv_lo + j * kTile + (tid + i * kThreads) / kChunks;
      page[i] = pos < unit.kv_hi ? __ldg(a.kv_indices + req.page0 + (pos >> shift)) : -1;
    }
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const int c = tid + i * kThreads;
      const int r = c / kChunks, ch = c % kChunks;
      const int pos = unit.kv_lo + j * kTile + r;
      const bool ok = page[i] >= 0;
      const size_t off = ok ? (((size_t)page[i] * P + (pos & (P - 1))) * Hk + unit.kv_head) * D + ch * 16 : 0;
      cp_async_16(kdst + r * D + ch * 16, a.k + off, ok ? 16u : 0u);
      cp_async_16(vdst + r * D + ch * 16, a.v + off, ok ? 16u : 0u);
    }
  };

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < n) load_tile(s, s);
    cp_async_commit();
  }

  // Q as f16 mma A fragments: rows = heads of the group (zero past G), k = head_dim.
  uint32_t qa[D / 16][4];
  {
    const int r0 = lane >> 2, kq = (lane & 3) * 2;
    const __nv_bfloat16* qrow = a.q + ((size_t)req.q_start * a.g.num_qo_heads + unit.kv_head * G) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      auto ld = [&](int row, int col) -> uint32_t {
        if (row >= G) return 0u;
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(qrow + (size_t)row * D + col);
        const float2 f = __bfloat1622float2(b);
        return pack_f16x2(f.x, f.y);
      };
      qa[kk][0] = ld(r0, kk * 16 + kq);
      qa[kk][1] = ld(r0 + 8, kk * 16 + kq);
      qa[kk][2] = ld(r0, kk * 16 + kq + 8);
      qa[kk][3] = ld(r0 + 8, kk * 16 + kq + 8);
    }
  }

  const float ks = a.k_scale ? a.k_scale[unit.kv_head] : 1.f;
  const float vs = a.v_scale ? a.v_scale[unit.kv_head] : 1.f;
  const float scale = a.g.sm_scale_log2 * ks;
  float o_acc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) o_acc[i][0] = o_acc[i][1] = o_acc[i][2] = o_acc[i][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows lane/4 and lane/4 + 8

  for (int j = 0; j < n; ++j) {
    cp_async_wait<kStages - 2>();
    __syncthreads();
    if (j + kStages - 1 < n) load_tile(j + kStages - 1, (j + kStages - 1) % kStages);
    cp_async_commit();

    // this warp's 16 keys of the tile: codes -> f16 rows (t = 0: K, t = 1: V)
    const uint32_t kcode = sbase + (j % kStages) * 2 * kCodeTile;
    auto convert = [&](int t) {
      const uint32_t src = kcode + t * kCodeTile;
#pragma unroll
      for (int c = lane; c < 16 * kChunks; c += 32) {
        const int r = warp * 16 + c / kChunks, ch = c % kChunks;
        const uint4 w = ld_shared_v4(src + r * D + ch * 16);
        st_shared_v4(f16t + f16_off<D>(r, 2 * ch), e4m3x2_to_f16x2(w.x), e4m3x2_to_f16x2(w.x >> 16),
                     e4m3x2_to_f16x2(w.y), e4m3x2_to_f16x2(w.y >> 16));
        st_shared_v4(f16t + f16_off<D>(r, 2 * ch + 1), e4m3x2_to_f16x2(w.z), e4m3x2_to_f16x2(w.z >> 16),
                     e4m3x2_to_f16x2(w.w), e4m3x2_to_f16x2(w.w >> 16));
      }
      __syncwarp();
    };
    convert(0);

    // S[16 x 16] = Q . K^T for this warp's 16 keys
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    {
      const int mi = lane >> 3;
      const int row = warp * 16 + (lane & 7) + (mi >> 1) * 8;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(f16t + f16_off<D>(row, kk * 2 + (mi & 1)), b0, b1, b2, b3);
        mma16816_f16(s[0], qa[kk], b0, b1);
        mma16816_f16(s[1], qa[kk], b2, b3);
      }
    }
    // mask keys past the unit's end, scale into the base-2 domain
    const int key0 = unit.kv_lo + j * kTile + warp * 16 + (lane & 3) * 2;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key0 + nt * 8 + (e & 1);
        s[nt][e] = key < unit.kv_hi ? s[nt][e] * scale : -INFINITY;
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
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      o_acc[i][0] *= a0;
      o_acc[i][1] *= a0;
      o_acc[i][2] *= a1;
      o_acc[i][3] *= a1;
    }
    __syncwarp();  // every lane's K fragments are read before V overwrites the rows
    convert(1);
    uint32_t pa[4];
    pa[0] = pack_f16x2(s[0][0], s[0][1]);
    pa[1] = pack_f16x2(s[0][2], s[0][3]);
    pa[2] = pack_f16x2(s[1][0], s[1][1]);
    pa[3] = pack_f16x2(s[1][2], s[1][3]);
    {
      const int mi = lane >> 3;
      const int row = warp * 16 + (lane & 7) + (mi & 1) * 8;
#pragma unroll
      for (int np = 0; np < D / 16; ++np) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(f16t + f16_off<D>(row, np * 2 + (mi >> 1)), b0, b1, b2, b3);
        mma16816_f16(o_acc[np * 2], pa, b0, b1);
        mma16816_f16(o_acc[np * 2 + 1], pa, b2, b3);
      }
    }
    __syncwarp();  // the next tile's conversion overwrites this warp's f16 rows
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
  const size_t pipe = (size_t)kStages * 2 * kTile * D + (size_t)kTile * D * 2;
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
