// Host planner: turns a batch's ragged query lengths and page table into a CTA
// work list (tiles of packed query rows x KV chunks) and a merge list for the
// requests whose KV is split across CTAs.
//
// FlashInfer 0.2 release, "Faster plan function": scheduling runs on the host
// from host arrays and its result reaches the device in one non-blocking copy.
// flashinfer-trace discussion #15, "Tunable Solutions and their Implementation
// Configs": split-KV is a scheduling knob (disable_split_kv) that must not
// change results beyond rounding.
#pragma once
#include <cstdint>
#include <string>
#include <vector>

#include "pkv_internal.h"

namespace pkv {

struct PlanInput {
  const int32_t* qo_indptr;         // host [batch+1]
  const int32_t* kv_indptr;         // host [batch+1]
  const int32_t* kv_last_page_len;  // host [batch]
  int32_t batch;
  int32_t num_qo_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t head_dim_v;
  int32_t head_dim_pe;  // > 0 selects MLA
  int32_t page_size;
  int32_t causal;
  float sm_scale;
  int32_t num_sms;
  int32_t disable_split_kv;
  int32_t kv_chunk;     // > 0 forces the split chunk
  int32_t kv_layout;    // 0 NHD, 1 HND (GQA/MHA pools)
  int32_t kv_fp8;       // 1: a decode plan for the FP8-KV kernel (sizes its split for that kernel)
};

struct Schedule {
  KernelKind kind = kKindPrefill;
  LaunchGeom geom{};
  std::vector<ReqInfo> reqs;
  std::vector<WorkUnit> units;
  std::vector<MergeTask> merges;
  std::vector<int32_t> cta_ptr;  // prefill: [num_ctas + 1] offsets of each CTA's units
  std::vector<int32_t> kv_row0;  // MLA prefill: [batch] first row of each request in the packed latent copy
  int32_t num_slots = 0;
  int32_t kv_chunk = 0;   // chunk used (0 = no split)
  int32_t num_sms = 0;
};

// Status codes mirror pkv_status: 0 ok, 1 invalid, 2 unsupported.
int build_schedule(const PlanInput& in, Schedule* out, std::string* err);

}  // namespace pkv
