// Host planner (see planner.h).
//
// Query rows are packed per kv head: for request b and kv head g, packed row
// r = t * group + i stands for token t of the request and qo head g*group + i.
// A tile is kBlockM consecutive packed rows, so with a large group (h16/kv1) a
// tile covers a few tokens of all heads that share one K/V stream, and every
// K/V tile the CTA loads is reused by all of its rows.
//
// With causal masking (bottom-right, see pkv.h) the last token of a tile bounds
// the keys the tile needs: keys [0, t_last + kv_len - qo_len + 1).
#include "planner.h"

#include <algorithm>
#include <cmath>
#include <functional>
#include <numeric>
#include <queue>
#include <utility>

namespace pkv {

namespace {

// K/V bytes above which prefill units are ordered in L2-sized bands (L2 is
// 126 MB on B200; Q, O and other CTAs' data share it).
constexpr int64_t kL2BandBytes = 48ll << 20;

bool is_pow2(int32_t x) { return x > 0 && (x & (x - 1)) == 0; }

int ilog2(int32_t x) {
  int s = 0;
  while ((1 << s) < x) ++s;
  return s;
}

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

struct Tile {
  int32_t req, kv_head, row0, rows, kv_need;
};

// Decode split model (GQA and MLA decode). What a split buys is balance: the
// units (tile x KV chunk) are taken longest first by `slots` resident CTAs,
// and the launch ends with its most loaded slot. Costs
// are in keys: a unit costs its keys plus kDecodeUnitCost (prologue, Q load,
// epilogue), and any split adds one merge launch, kDecodeMergeCost. Both
// constants were fitted to measured launch times of decode batches on B200
// (the model ranks chunk lengths as the measurements did; without the merge
// cost it prefers splits that measured slower than none).
constexpr int64_t kDecodeUnitCost = 256;
constexpr int64_t kDecodeMergeCost = 400;

// Makespan, in keys, of the units that chunk length `c` (0 = no split) cuts the
// tiles into, when `slots` CTAs take them longest first. Full chunks all have
// length c and are the longest units, so they are dealt round-robin; the
// remainders (one per tile at most) go, longest first, to the least loaded
// slot. `need` is sorted in descending order; `rem` and `heap` are scratch.
int64_t decode_makespan(const std::vector<int64_t>& need, int64_t c, int64_t slots, std::vector<int64_t>& rem,
                        std::vector<int64_t>& heap) {
  int64_t full = 0;
  rem.clear();
  size_t whole = 0;  // need[whole..] fit one chunk and keep their sorted order
  if (c > 0) {
    while (whole < need.size() && need[whole] > c) {
      full += need[whole] / c;
      if (need[whole] % c) rem.push_back(need[whole] % c);
      ++whole;
    }
    std::sort(rem.begin(), rem.end(), std::greater<int64_t>());
  }
  const int64_t k = full / slots, extra = full % slots;
  heap.clear();
  int64_t worst = 0;
  for (int64_t i = 0; i < slots; ++i) {
    const int64_t l = (k + (i < extra ? 1 : 0)) * (c + kDecodeUnitCost);
    heap.push_back(l);
    worst = std::max(worst, l);
  }
  std::make_heap(heap.begin(), heap.end(), std::greater<int64_t>());
  auto place = [&](int64_t r) {
    std::pop_heap(heap.begin(), heap.end(), std::greater<int64_t>());
    heap.back() += r + kDecodeUnitCost;
    worst = std::max(worst, heap.back());
    std::push_heap(heap.begin(), heap.end(), std::greater<int64_t>());
  };
  // longest first: merge the sorted remainders with the sorted whole tiles
  size_t i = 0, j = whole;
  while (i < rem.size() || j < need.size()) {
    if (j == need.size() || (i < rem.size() && rem[i] >= need[j])) place(rem[i++]);
    else place(need[j++]);
  }
  return worst;
}

// Resident CTAs per SM of the decode kernels on sm_100a (set by their shared
// memory and registers): GQA with bf16 K/V 2 at head_dim 128, the FP8 kernel 3,
// either 4 at head_dim 64; MLA decode 2.
int64_t decode_ctas_per_sm(KernelKind kind, int32_t head_dim, bool fp8) {
  if (kind == kKindMlaDecode) return 2;
  return head_dim <= 64 ? 4 : fp8 ? 3 : 2;
}

}  // namespace

int build_schedule(const PlanInput& in, Schedule* out, std::string* err) {
  Schedule s;
  const bool mla = in.head_dim_pe > 0;
  if (in.batch < 0) { *err = "batch < 0"; return 1; }
  if (in.batch > 0 && (!in.qo_indptr || !in.kv_indptr || !in.kv_last_page_len)) {
    *err = "NULL indptr / last_page_len"; return 1;
  }
  if (in.num_qo_heads <= 0 || in.num_kv_heads <= 0) { *err = "head counts must be positive"; return 1; }
  if (in.num_qo_heads % in.num_kv_heads != 0) { *err = "num_qo_heads % num_kv_heads != 0"; return 1; }
  if (in.kv_layout != 0 && in.kv_layout != 1) { *err = "kv_layout must be 0 (NHD) or 1 (HND)"; return 1; }
  if (!is_pow2(in.page_size) || in.page_size > 256) {
    *err = "page_size must be a power of two in [1, 256]"; return 2;
  }
  if (!std::isfinite(in.sm_scale)) { *err = "sm_scale is not finite"; return 1; }
  if (!(in.sm_scale > 0.f)) { *err = "sm_scale must be positive"; return 2; }
  const int32_t group = in.num_qo_heads / in.num_kv_heads;
  if (mla) {
    if (in.num_kv_heads != 1 || in.head_dim != 512 || in.head_dim_v != 512 || in.head_dim_pe != 64) {
      *err = "MLA supports head_dim_ckv 512, head_dim_kpe 64, one latent head"; return 2;
    }
    if (in.num_qo_heads > 128) { *err = "MLA supports at most 128 heads"; return 2; }
  } else {
    if (in.head_dim != 64 && in.head_dim != 128) { *err = "head_dim must be 64 or 128"; return 2; }
    if (in.head_dim_v != in.head_dim) { *err = "head_dim_v must equal head_dim"; return 2; }
    if (group > 128) { *err = "group size num_qo_heads / num_kv_heads must be <= 128"; return 2; }
  }

  // ---- validate the page table, build per-request info
  if (in.batch > 0) {
    if (in.qo_indptr[0] != 0 || in.kv_indptr[0] != 0) { *err = "indptr must start at 0"; return 1; }
  }
  s.reqs.resize(in.batch);
  int32_t max_qo = 0;
  for (int32_t b = 0; b < in.batch; ++b) {
    const int32_t qo = in.qo_indptr[b + 1] - in.qo_indptr[b];
    const int32_t np = in.kv_indptr[b + 1] - in.kv_indptr[b];
    if (qo < 0) { *err = "qo_indptr is not non-decreasing"; return 1; }
    if (np < 0) { *err = "kv_indptr is not non-decreasing"; return 1; }
    const int32_t last = in.kv_last_page_len[b];
    if (np > 0 && (last < 1 || last > in.page_size)) {
      *err = "kv_last_page_len must be in [1, page_size] for a request with pages"; return 1;
    }
    const int64_t kv_len = np > 0 ? (int64_t)(np - 1) * in.page_size + last : 0;
    if (kv_len > INT32_MAX / 2) { *err = "kv_len too large"; return 2; }
    if ((int64_t)qo * group > INT32_MAX / 2) { *err = "qo_len * group too large"; return 2; }
    s.reqs[b] = ReqInfo{in.qo_indptr[b], qo, (int32_t)kv_len, in.kv_indptr[b]};
    max_qo = std::max(max_qo, qo);
  }

  // ---- kernel choice
  if (mla) s.kind = (max_qo <= 1 && in.num_qo_heads <= kDecodeRows) ? kKindMlaDecode : kKindMla;
  else if (max_qo <= 1 && group <= kDecodeRows) s.kind = kKindDecode;
  else s.kind = kKindPrefill;

  // MLA prefill streams each request's latent rows from a packed, contiguous
  // copy (ckv | kpe per key, in key order) that the run builds first; only
  // requests with queries are packed.
  int64_t packed_rows = 0;
  int32_t max_kv = 0;
  for (int32_t b = 0; b < in.batch; ++b) max_kv = std::max(max_kv, s.reqs[b].kv_len);
  if (s.kind == kKindMla) {
    s.kv_row0.assign(in.batch, 0);
    for (int32_t b = 0; b < in.batch; ++b) {
      s.kv_row0[b] = (int32_t)std::min<int64_t>(packed_rows, INT32_MAX);
      if (s.reqs[b].qo_len > 0) packed_rows += s.reqs[b].kv_len;
    }
    if (packed_rows > INT32_MAX / 2) { *err = "MLA prefill: more than 2^30 keys in one batch"; return 2; }
  }

  const int32_t num_sms = in.num_sms > 0 ? in.num_sms : 148;
  s.num_sms = num_sms;
  // Rows per work unit: decode packs one token's group of heads into an mma.sync
  // tile; prefill units hold two 128-row tensor-core tiles that share K/V; MLA
  // packs tokens x heads the same way with one latent "kv head".
  const int32_t rows_per_tile = (s.kind == kKindDecode || s.kind == kKindMlaDecode) ? kDecodeRows
                                : s.kind == kKindMla  ? kMlaUnitRows
                                                      : kPrefillUnitRows;

  // ---- tiles
  std::vector<Tile> tiles;
  int64_t total_cost = 0;
  int32_t max_need = 0;
  for (int32_t b = 0; b < in.batch; ++b) {
    const ReqInfo& r = s.reqs[b];
    const int64_t packed = (int64_t)r.qo_len * group;
    for (int32_t g = 0; g < in.num_kv_heads; ++g) {
      for (int64_t row0 = 0; row0 < packed; row0 += rows_per_tile) {
        const int32_t rows = (int32_t)std::min<int64_t>(rows_per_tile, packed - row0);
        const int64_t t_last = (row0 + rows - 1) / group;
        int64_t need = r.kv_len;
        if (in.causal) need = std::min<int64_t>(r.kv_len, std::max<int64_t>(0, t_last + r.kv_len - r.qo_len + 1));
        tiles.push_back(Tile{b, g, (int32_t)row0, rows, (int32_t)need});
        total_cost += need + 64;
        max_need = std::max<int32_t>(max_need, (int32_t)need);
      }
    }
  }

  // ---- split-KV chunk
  const int32_t align = (s.kind == kKindDecode || s.kind == kKindMlaDecode) ? kDecodeTileN
                        : s.kind == kKindMla                               ? 64
                                                                           : kBlockN;
  int64_t chunk = 0;  // 0 = no split
  if (!in.disable_split_kv) {
    if (in.kv_chunk > 0) {
      chunk = round_up(in.kv_chunk, align);
    } else if (s.kind == kKindDecode || s.kind == kKindMlaDecode) {
      // Candidates from half the average load per slot up to the longest tile
      // (x1.15 steps), and no split; the cheapest by decode_makespan wins.
      // When no tile reaches half the average load, longest-first placement of
      // whole tiles is already balanced: no split, and no search.
      const int64_t slots = decode_ctas_per_sm(s.kind, in.head_dim, in.kv_fp8 != 0) * (int64_t)num_sms;
      std::vector<int64_t> need, rem, heap;
      need.reserve(tiles.size());
      int64_t total = 0;
      for (const Tile& t : tiles) {
        need.push_back(t.kv_need);
        total += t.kv_need + kDecodeUnitCost;
      }
      std::sort(need.begin(), need.end(), std::greater<int64_t>());
      const int64_t avg = total / std::max<int64_t>(1, slots);
      if ((int64_t)max_need * 2 <= avg) {
        chunk = 0;
      } else if (tiles.size() > 8192) {
        chunk = round_up(std::max<int64_t>(avg, 4 * align), align);  // too many tiles to search cheaply
      } else {
        int64_t best = 0, best_t = decode_makespan(need, 0, slots, rem, heap);
        for (int64_t c = std::max<int64_t>(4 * align, round_up(avg / 2, align)); c < max_need;
             c = std::max<int64_t>(c + align, (c * 115 / 100) / align * align)) {
          const int64_t t_est = decode_makespan(need, c, slots, rem, heap) + kDecodeMergeCost;
          if (t_est < best_t) {
            best_t = t_est;
            best = c;
          }
        }
        chunk = best;
      }
    } else {
      // Prefill: one CTA per SM at a time; split only when a single tile is
      // longer than the average work per SM.
      chunk = round_up(std::max<int64_t>(256, (total_cost + num_sms - 1) / num_sms), align);
    }
    if (chunk >= max_need) chunk = 0;
  }
  s.kv_chunk = (int32_t)chunk;

  // ---- units and merges
  int32_t slots = 0;
  for (const Tile& t : tiles) {
    if (chunk == 0 || t.kv_need <= chunk) {
      s.units.push_back(WorkUnit{t.req, t.kv_head, t.row0, t.rows, 0, t.kv_need, -1, 0});
      continue;
    }
    const int32_t n = (int32_t)((t.kv_need + chunk - 1) / chunk);
    s.merges.push_back(MergeTask{t.req, t.kv_head, t.row0, t.rows, slots, n, 0, 0});
    for (int32_t c = 0; c < n; ++c) {
      const int32_t lo = (int32_t)(c * chunk);
      const int32_t hi = (int32_t)std::min<int64_t>(t.kv_need, (int64_t)(c + 1) * chunk);
      s.units.push_back(WorkUnit{t.req, t.kv_head, t.row0, t.rows, lo, hi, slots + c, 0});
    }
    slots += n;
  }
  s.num_slots = slots;

  // Longest units first: with a non-persistent grid the hardware hands out
  // CTAs roughly in index order, and the persistent prefill schedule below
  // assigns units in list order, so this is a greedy longest-processing-time
  // schedule that keeps the tail short.
  auto longest_first = [](const WorkUnit& a, const WorkUnit& b) {
    return (a.kv_hi - a.kv_lo) > (b.kv_hi - b.kv_lo);
  };
  int64_t kv_bytes = 0;  // K and V bytes of the whole batch
  for (const ReqInfo& r : s.reqs) kv_bytes += (int64_t)r.kv_len * in.num_kv_heads * (in.head_dim + in.head_dim_v) * 2;
  if (s.kind == kKindPrefill && kv_bytes > kL2BandBytes) {
    // When the batch's K/V does not fit in L2 beside everything else, a global
    // longest-first order runs one unit of every (request, kv head) at a time
    // and each unit re-reads its keys from HBM. Instead cut the work list (in
    // (request, kv head) order) into bands of whole groups holding at least
    // one unit per SM, longest first within a band: the units that run at the
    // same time then share a few groups' K/V, which stays in L2.
    std::vector<WorkUnit> out;
    out.reserve(s.units.size());
    size_t begin = 0;
    while (begin < s.units.size()) {
      size_t end = begin;
      while (end < s.units.size()) {
        const WorkUnit& u = s.units[end];
        ++end;
        const bool group_ends = end == s.units.size() || s.units[end].req != u.req || s.units[end].kv_head != u.kv_head;
        if (group_ends && end - begin >= (size_t)num_sms) break;
      }
      std::stable_sort(s.units.begin() + begin, s.units.begin() + end, longest_first);
      out.insert(out.end(), s.units.begin() + begin, s.units.begin() + end);
      begin = end;
    }
    s.units.swap(out);
  } else {
    std::stable_sort(s.units.begin(), s.units.end(), longest_first);
  }

  // Prefill and MLA prefill run persistent CTAs (one per SM), each over a
  // fixed list of units. Greedy list scheduling in the longest-first order
  // above: each unit goes to the CTA with the least work so far, counted in
  // keys of whole KV tiles of the kernel plus the unit's own start and end:
  // one 128-key tile for the prefill, two and a half 32-key tiles for the MLA
  // prefill, whose unit boundary (the next unit's Q load and this unit's
  // output) measured that long in a clock64 trace. The units are then stored
  // CTA by CTA.
  int32_t num_ctas = (int32_t)s.units.size();
  if ((s.kind == kKindPrefill || s.kind == kKindMla) && !s.units.empty()) {
    const int64_t tile = s.kind == kKindMla ? kMlaTileN : kBlockN;
    const int64_t edge = s.kind == kKindMla ? 5 * kMlaTileN / 2 : kBlockN;
    num_ctas = (int32_t)std::min<size_t>((size_t)num_sms, s.units.size());
    using Load = std::pair<int64_t, int32_t>;  // (work so far, cta)
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int32_t c = 0; c < num_ctas; ++c) heap.push({0, c});
    std::vector<std::vector<WorkUnit>> lists((size_t)num_ctas);
    for (const WorkUnit& u : s.units) {
      Load top = heap.top();
      heap.pop();
      lists[(size_t)top.second].push_back(u);
      top.first += (u.kv_hi - u.kv_lo + tile - 1) / tile * tile + edge;
      heap.push(top);
    }
    s.units.clear();
    s.cta_ptr.assign(1, 0);
    for (const auto& l : lists) {
      s.units.insert(s.units.end(), l.begin(), l.end());
      s.cta_ptr.push_back((int32_t)s.units.size());
    }
  }

  LaunchGeom& gm = s.geom;
  gm.num_qo_heads = in.num_qo_heads;
  gm.num_kv_heads = in.num_kv_heads;
  gm.group = group;
  gm.head_dim = in.head_dim;
  gm.head_dim_v = in.head_dim_v;
  gm.head_dim_pe = in.head_dim_pe;
  gm.page_size = in.page_size;
  gm.page_shift = ilog2(in.page_size);
  gm.causal = in.causal ? 1 : 0;
  gm.sm_scale_log2 = (float)((double)in.sm_scale * 1.4426950408889634);
  gm.part_rows = rows_per_tile;
  gm.num_units = (int32_t)s.units.size();
  gm.num_merge = (int32_t)s.merges.size();
  gm.total_q = in.batch > 0 ? in.qo_indptr[in.batch] : 0;
  gm.num_ctas = num_ctas;
  gm.kv_layout = mla ? 0 : in.kv_layout;  // a latent pool has no head axis: both layouts coincide
  gm.packed_rows = (int32_t)packed_rows;
  gm.max_kv_len = max_kv;
  gm.num_reqs = in.batch;
  *out = std::move(s);
  return 0;
}

}  // namespace pkv
