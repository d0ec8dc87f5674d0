// Data shared by the host planner and the kernels: the work list a plan
// uploads into the caller's workspace and the parameter blocks the launchers
// pass. Plain structs of int32 so the host writes them byte for byte.
#pragma once
#include <cstddef>
#include <cstdint>

namespace pkv {

constexpr int kBlockM = 128;   // packed (token, head-in-group) rows per tensor-core tile (TMEM lanes)
constexpr int kPrefillUnitRows = 256;  // packed rows per prefill work unit (two tiles share K/V)
constexpr int kMlaUnitRows = 64;       // packed (token, head) rows per MLA work unit (M = 64 MMAs)
constexpr int kMlaTileN = 32;          // latent keys per MLA prefill tile
constexpr int kBlockN = 128;   // KV slots per prefill KV tile
constexpr int kDecodeRows = 16;  // packed rows per decode unit (mma.sync M)
constexpr int kDecodeTileN = 64;  // KV slots per decode pipeline stage

enum KernelKind : int32_t { kKindPrefill = 0, kKindDecode = 1, kKindMla = 2, kKindMlaDecode = 3 };

// One CTA's worth of attention: packed query rows [row0, row0 + rows) of
// request `req` for kv head `kv_head`, over keys [kv_lo, kv_hi).
// `partial` < 0: write O / LSE straight to the outputs; otherwise write fp32
// partial state into partial slot `partial` for a later merge.
struct WorkUnit {
  int32_t req;
  int32_t kv_head;
  int32_t row0;
  int32_t rows;
  int32_t kv_lo;
  int32_t kv_hi;
  int32_t partial;
  int32_t pad;
};
static_assert(sizeof(WorkUnit) == 32, "WorkUnit is 32 bytes");

// Merge of `num` consecutive partial slots starting at `slot0` into packed rows
// [row0, row0 + rows) of request `req`, kv head `kv_head`.
struct MergeTask {
  int32_t req;
  int32_t kv_head;
  int32_t row0;
  int32_t rows;
  int32_t slot0;
  int32_t num;
  int32_t pad0;
  int32_t pad1;
};
static_assert(sizeof(MergeTask) == 32, "MergeTask is 32 bytes");

// Per-request metadata copied to the device: qo start, qo_len, kv_len, first page.
struct ReqInfo {
  int32_t q_start;
  int32_t qo_len;
  int32_t kv_len;
  int32_t page0;   // offset of the request's first entry in kv_indices
};
static_assert(sizeof(ReqInfo) == 16, "ReqInfo is 16 bytes");

// Everything a launch needs besides the user's tensors.
struct LaunchGeom {
  int32_t num_qo_heads;
  int32_t num_kv_heads;
  int32_t group;          // num_qo_heads / num_kv_heads
  int32_t head_dim;       // QK width (ckv width for MLA)
  int32_t head_dim_v;
  int32_t head_dim_pe;    // MLA rope width, 0 otherwise
  int32_t page_size;
  int32_t page_shift;     // log2(page_size)
  int32_t causal;
  float sm_scale_log2;    // sm_scale * log2(e)
  int32_t part_rows;      // rows per partial slot
  int32_t num_units;
  int32_t num_merge;
  int32_t total_q;        // rows of q (tokens)
  int32_t num_ctas;       // CTAs of the main launch (prefill: persistent, one unit list each)
  int32_t kv_layout;      // 0 NHD [page, slot, kv head, D]; 1 HND [page, kv head, slot, D]
  int32_t packed_rows;    // MLA prefill: rows of the packed latent copy (sum of kv_len of requests with queries)
  int32_t max_kv_len;     // longest kv_len of the batch
  int32_t num_reqs;       // requests (batch)
};

// Device pointers into the workspace after upload.
struct DeviceView {
  const WorkUnit* units;
  const MergeTask* merges;
  const ReqInfo* reqs;
  float* part_o;          // [num_slots, part_rows, head_dim_v]
  float* part_lse;        // [num_slots, part_rows]
  int* status;            // device status word (0 = ok)
  const int32_t* cta_ptr; // prefill: CTA b runs units [cta_ptr[b], cta_ptr[b + 1])
  const int32_t* kv_row0; // MLA prefill: first row of each request in the packed latent copy
  void* packed;           // MLA prefill: packed latent rows [packed_rows][ckv | kpe] bf16
};

}  // namespace pkv
