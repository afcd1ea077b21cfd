// C-ABI entry points of librk.so: argument validation, workspace layout,
// tensor-map set-up and kernel launches.  Every check that can be done on the
// host is done here, synchronously, before any GPU work is enqueued.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "rk_internal.h"

namespace rk {

cudaError_t launch_select(LayoutView* lv_dev, int n_tables, const rk_visible& vis, WsHeader* hdr,
                          Item* items_tmp, Item* items, int32_t* cursor, int64_t n_items,
                          cudaStream_t stream);
cudaError_t launch_relocate(const void* k_src, void* k_dst, const int32_t* jobs, int n_jobs,
                            int64_t n_src_pages, int64_t n_dst_pages, int P, int D, double theta,
                            int* device_error, cudaStream_t stream);

cudaError_t launch_prefill_args(const PrefillLaunchArgs& a, cudaStream_t stream);
cudaError_t launch_selftest_wait(int* word, int wait_ms, cudaStream_t stream);
cudaError_t launch_select_tables_only(LayoutView* lv_dev, int n_tables, const rk_visible& vis,
                                      WsHeader* hdr, cudaStream_t stream);

namespace {

constexpr int64_t kMaxI32 = 2147483647;

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

rk_status check_dims(const rk_dims* d) {
  if (!d) return RK_ERR_INVALID_ARG;
  if (d->n_req < 1 || d->n_layers < 1 || d->num_kv_heads < 1 || d->num_q_heads < 1)
    return RK_ERR_INVALID_ARG;
  if (d->num_q_heads % d->num_kv_heads != 0) return RK_ERR_INVALID_ARG;
  if (d->head_dim != 64 && d->head_dim != 128) return RK_ERR_INVALID_ARG;
  if (d->page_size != 16 && d->page_size != 64) return RK_ERR_INVALID_ARG;
  if (d->n_pages < 1 || d->n_pages * d->page_size + kKeysPerTile >= kMaxI32)
    return RK_ERR_INVALID_ARG;
  if (d->total_tokens < 0 || d->reserved != 0) return RK_ERR_INVALID_ARG;
  if (static_cast<int64_t>(d->n_layers) * d->total_tokens + kRowsPerTile >= kMaxI32)
    return RK_ERR_INVALID_ARG;
  return RK_OK;
}

// Everything derived from a validated layout.
struct Derived {
  int64_t n_tables = 0, n_lh = 0, total_pages = 0;
  int64_t entry_capacity = 0, range_capacity = 0, item_capacity = 0;
  std::vector<int32_t> seg_indptr, page_prefix;
  bool any_retrieval = false;
  int64_t n_retr = 0;
  WsMap map;
  int32_t layout_words = 0;
};

rk_status check_layout(const rk_dims* d, const rk_layout* lay, Derived* out) {
  if (!lay) return RK_ERR_INVALID_ARG;
  if (lay->n_segments < 0) return RK_ERR_INVALID_ARG;
  if ((lay->n_segments > 0 && (!lay->segments || !lay->page_base)) || !lay->cu_seqlens ||
      !lay->class_map || !lay->class_window)
    return RK_ERR_INVALID_ARG;
  const int n_req = d->n_req, P = d->page_size;
  const int64_t n_lh = static_cast<int64_t>(d->n_layers) * d->num_kv_heads;
  out->n_lh = n_lh;
  out->n_tables = n_lh * n_req;
  if (out->n_tables >= kMaxI32 / 4) return RK_ERR_INVALID_ARG;
  const int32_t* cu = lay->cu_seqlens;
  if (cu[0] != 0) return RK_ERR_INVALID_ARG;
  for (int r = 0; r < n_req; ++r)
    if (cu[r + 1] < cu[r]) return RK_ERR_INVALID_ARG;
  if (cu[n_req] != d->total_tokens) return RK_ERR_INVALID_ARG;
  bool any_local = false;
  for (int64_t k = 0; k < n_lh; ++k) {
    const int c = lay->class_map[k];
    if (c < RK_GLOBAL || c > RK_DENSE) return RK_ERR_INVALID_ARG;
    any_local |= c == RK_LOCAL;
    out->any_retrieval |= c == RK_RETRIEVAL;
  }
  if (any_local && lay->class_window[RK_LOCAL] < 1) return RK_ERR_INVALID_ARG;
  // segments: grouped by request, tiling [0, L_r) in order
  out->seg_indptr.assign(n_req + 1, 0);
  int prev_req = -1, expect = 0;
  for (int s = 0; s < lay->n_segments; ++s) {
    const rk_segment& g = lay->segments[s];
    if (g.req < 0 || g.req >= n_req || g.len < 1 || (g.cached != 0 && g.cached != 1))
      return RK_ERR_INVALID_ARG;
    if (g.req != prev_req) {
      if (g.req < prev_req) return RK_ERR_INVALID_ARG;
      if (prev_req >= 0 && expect != cu[prev_req + 1] - cu[prev_req]) return RK_ERR_INVALID_ARG;
      for (int r = prev_req + 1; r < g.req; ++r)
        if (cu[r + 1] != cu[r]) return RK_ERR_INVALID_ARG;  // skipped request must be empty
      prev_req = g.req;
      expect = 0;
    }
    if (g.logical_start != expect) return RK_ERR_INVALID_ARG;
    const int L = cu[g.req + 1] - cu[g.req];
    if (static_cast<int64_t>(g.logical_start) + g.len > L) return RK_ERR_INVALID_ARG;
    const int64_t delta = static_cast<int64_t>(g.logical_start) - g.stored_pos_base;
    if (g.cached && (delta > kMaxI32 || delta < -kMaxI32)) return RK_ERR_INVALID_ARG;
    const bool last = g.logical_start + g.len == L;
    if (!last && g.len % P != 0) return RK_ERR_UNALIGNED;
    const int64_t npg = (g.len + P - 1) / P;
    for (int64_t lh = 0; lh < n_lh; ++lh) {
      const int64_t b = lay->page_base[s * n_lh + lh];
      if (b < 0 || b + npg > d->n_pages) return RK_ERR_INVALID_ARG;
    }
    expect += g.len;
    out->seg_indptr[g.req + 1] = s + 1;
  }
  if (prev_req >= 0 && expect != cu[prev_req + 1] - cu[prev_req]) return RK_ERR_INVALID_ARG;
  for (int r = prev_req + 1; r < n_req; ++r)
    if (cu[r + 1] != cu[r]) return RK_ERR_INVALID_ARG;
  for (int r = 0; r < n_req; ++r)  // empty requests keep their predecessor's end
    if (out->seg_indptr[r + 1] < out->seg_indptr[r]) out->seg_indptr[r + 1] = out->seg_indptr[r];
  // retrieval lists
  if (out->any_retrieval && !lay->retr_indptr) return RK_ERR_INVALID_ARG;
  if (lay->retr_indptr) {
    if (lay->retr_indptr[0] != 0) return RK_ERR_INVALID_ARG;
    for (int64_t t = 0; t < out->n_tables; ++t)
      if (lay->retr_indptr[t + 1] < lay->retr_indptr[t]) return RK_ERR_INVALID_ARG;
    out->n_retr = lay->retr_indptr[out->n_tables];
    if (out->n_retr > 0 && !lay->retr_pages) return RK_ERR_INVALID_ARG;
    if (out->n_retr >= kMaxI32 / 4) return RK_ERR_INVALID_ARG;
  }
  // sizes
  out->page_prefix.assign(n_req + 1, 0);
  const int G = d->num_q_heads / d->num_kv_heads;
  const int64_t npairs = (G + 1) / 2;
  int64_t items = 0;
  for (int r = 0; r < n_req; ++r) {
    const int64_t L = cu[r + 1] - cu[r];
    out->page_prefix[r + 1] =
        static_cast<int32_t>(out->page_prefix[r] + (L + P - 1) / P);
    const int64_t nseg = out->seg_indptr[r + 1] - out->seg_indptr[r];
    items += n_lh * npairs * (L / kRowsPerTile + 1 + nseg);
  }
  out->total_pages = out->page_prefix[n_req];
  out->entry_capacity = n_lh * out->total_pages;
  out->range_capacity = n_lh * lay->n_segments;
  out->item_capacity = items;
  if (out->entry_capacity >= kMaxI32 || out->range_capacity >= kMaxI32 ||
      out->item_capacity >= kMaxI32 / 2)
    return RK_ERR_INVALID_ARG;
  // workspace map
  const int64_t words_fixed = (sizeof(LayoutView) + 3) / 4;
  const int64_t words = words_fixed + 5 * static_cast<int64_t>(lay->n_segments) + (n_req + 1) +
                        lay->n_segments * n_lh + (n_req + 1) + (n_req + 1) + n_lh +
                        (out->n_tables + 1) + out->n_retr + (out->n_tables + 1) + kCostBuckets + 8;
  if (words >= kMaxI32) return RK_ERR_INVALID_ARG;
  out->layout_words = static_cast<int32_t>(words);
  WsMap& m = out->map;
  m.header = 0;
  m.items = sizeof(WsHeader);
  m.items_tmp = align_up(m.items + sizeof(Item) * out->item_capacity, 256);
  m.cursor = align_up(m.items_tmp + sizeof(Item) * out->item_capacity, 256);
  m.layout = align_up(m.cursor + 4 * static_cast<size_t>(kCostBuckets), 256);
  m.total = align_up(m.layout + 4 * static_cast<size_t>(words), 256);
  return RK_OK;
}

// Host image of the workspace's header + layout block.
void build_layout_image(const rk_dims* d, const rk_layout* lay, const Derived& dv,
                        std::vector<int32_t>* img) {
  img->assign(dv.layout_words, 0);
  LayoutView v{};
  v.n_req = d->n_req;
  v.n_layers = d->n_layers;
  v.hq = d->num_q_heads;
  v.hkv = d->num_kv_heads;
  v.d = d->head_dim;
  v.p = d->page_size;
  v.n_seg = lay->n_segments;
  v.n_retr = static_cast<int32_t>(dv.n_retr);
  v.n_pages = d->n_pages;
  v.total_tokens = d->total_tokens;
  v.total_pages = static_cast<int32_t>(dv.total_pages);
  v.window = lay->class_window[RK_LOCAL];
  v.item_capacity = static_cast<int32_t>(dv.item_capacity);
  int32_t max_pages = 0;
  for (int r = 0; r < d->n_req; ++r)
    max_pages = std::max(max_pages, dv.page_prefix[r + 1] - dv.page_prefix[r]);
  v.max_table_pages = max_pages;
  {
    // work-list groups: (request, layer) pairs, a power of two of them so
    // that each gets an equal share of the cost buckets; past
    // kMaxBucketGroups one group (plain longest-first order)
    const int64_t n_groups = static_cast<int64_t>(d->n_req) * d->n_layers;
    int groups = 1;
    if (n_groups > 1 && n_groups <= kMaxBucketGroups)
      while (groups < n_groups) groups <<= 1;
    const int bpg = kCostBuckets / groups;
    const int ept = kKeysPerTile / d->page_size;
    const int max_cost = (max_pages + ept - 1) / ept + 1;
    v.bucket_groups = groups;
    v.cost_width = std::max(1, (max_cost + 1 + bpg - 1) / bpg);
  }
  int32_t off = static_cast<int32_t>((sizeof(LayoutView) + 3) / 4);
  int32_t* w = img->data();
  v.off_seg = off;
  for (int s = 0; s < lay->n_segments; ++s) {
    const rk_segment& g = lay->segments[s];
    w[off + 5 * s + 0] = g.req;
    w[off + 5 * s + 1] = g.logical_start;
    w[off + 5 * s + 2] = g.len;
    w[off + 5 * s + 3] = g.cached ? g.stored_pos_base : g.logical_start;
    w[off + 5 * s + 4] = g.cached;
  }
  off += 5 * lay->n_segments;
  v.off_seg_indptr = off;
  for (int r = 0; r <= d->n_req; ++r) w[off + r] = dv.seg_indptr[r];
  off += d->n_req + 1;
  v.off_page_base = off;
  if (lay->n_segments > 0)
    std::memcpy(w + off, lay->page_base, 4 * static_cast<size_t>(lay->n_segments) * dv.n_lh);
  off += static_cast<int32_t>(lay->n_segments * dv.n_lh);
  v.off_cu = off;
  for (int r = 0; r <= d->n_req; ++r) w[off + r] = lay->cu_seqlens[r];
  off += d->n_req + 1;
  v.off_page_prefix = off;
  for (int r = 0; r <= d->n_req; ++r) w[off + r] = dv.page_prefix[r];
  off += d->n_req + 1;
  v.off_class = off;
  for (int64_t k = 0; k < dv.n_lh; ++k) w[off + k] = lay->class_map[k];
  off += static_cast<int32_t>(dv.n_lh);
  v.off_retr_indptr = off;
  for (int64_t t = 0; t <= dv.n_tables; ++t) w[off + t] = lay->retr_indptr ? lay->retr_indptr[t] : 0;
  off += static_cast<int32_t>(dv.n_tables + 1);
  v.off_retr_pages = off;
  if (dv.n_retr > 0) std::memcpy(w + off, lay->retr_pages, 4 * static_cast<size_t>(dv.n_retr));
  off += static_cast<int32_t>(dv.n_retr);
  // work items per table (the attention work list's shape, known from the
  // layout): <= 128-row tiles of the table's row set x pairs of q heads; the
  // row set follows the class rule that the select kernel also applies
  // (global / dense: the whole request; local / retrieval: the uncached
  // segments, adjacent ones merged)
  v.off_tile_prefix = off;
  {
    const int G = d->num_q_heads / d->num_kv_heads;
    const int npairs = (G + 1) / 2;
    int64_t acc = 0;
    for (int r = 0; r < d->n_req; ++r) {
      const int L = lay->cu_seqlens[r + 1] - lay->cu_seqlens[r];
      int all_tiles = (L + kRowsPerTile - 1) / kRowsPerTile;
      int unc_tiles = 0;
      for (int sg = dv.seg_indptr[r], cur_b = -1, cur_e = -1; sg <= dv.seg_indptr[r + 1]; ++sg) {
        const bool end = sg == dv.seg_indptr[r + 1];
        const bool unc = !end && !lay->segments[sg].cached;
        const int a = end ? 0 : lay->segments[sg].logical_start;
        if (unc && cur_e == a) {
          cur_e = a + lay->segments[sg].len;
          continue;
        }
        if (cur_e > cur_b) unc_tiles += (cur_e - cur_b + kRowsPerTile - 1) / kRowsPerTile;
        cur_b = cur_e = -1;
        if (unc) {
          cur_b = a;
          cur_e = a + lay->segments[sg].len;
        }
      }
      for (int layer = 0; layer < d->n_layers; ++layer)
        for (int h = 0; h < d->num_kv_heads; ++h) {
          const int t = (r * d->n_layers + layer) * d->num_kv_heads + h;
          const int cls = lay->class_map[layer * d->num_kv_heads + h];
          w[off + t] = static_cast<int32_t>(acc);
          acc += static_cast<int64_t>(npairs) *
                 ((cls == RK_GLOBAL || cls == RK_DENSE) ? all_tiles : unc_tiles);
        }
    }
    w[off + dv.n_tables] = static_cast<int32_t>(acc);
  }
  off += static_cast<int32_t>(dv.n_tables + 1);
  v.off_cost_hist = off;  // zero: the select kernel's CTAs add their items' costs
  off += kCostBuckets;
  v.layout_words = off;
  std::memcpy(w, &v, sizeof(LayoutView));
}

// ---- retrieval page scoring: the host image the scoring kernels read

struct ScorePlan {
  std::vector<int32_t> img;  // ScoreView followed by its arrays
  ScoreView sv{};
  int64_t max_pages = 0;     // pages of the longest request (scores row length)
  size_t off_partials = 0, off_kbar = 0, off_urot = 0, total = 0;  // workspace offsets
};

// A copy of the layout whose retrieval lists are empty when it has none:
// scoring produces the lists, so it must accept a layout without them.
struct ScoreLayout {
  rk_layout lay;
  std::vector<int32_t> empty_indptr;
};

void score_layout(const rk_dims* d, const rk_layout* in, ScoreLayout* out) {
  out->lay = *in;
  if (!in->retr_indptr) {
    const int64_t n_tables = static_cast<int64_t>(d->n_req) * d->n_layers * d->num_kv_heads;
    out->empty_indptr.assign(static_cast<size_t>(n_tables + 1), 0);
    out->lay.retr_indptr = out->empty_indptr.data();
    out->lay.retr_pages = nullptr;
  }
}

rk_status build_score_plan(const rk_dims* d, const rk_layout* lay, const Derived& dv,
                           int top_k, ScorePlan* out) {
  const int P = d->page_size, D = d->head_dim, n_req = d->n_req;
  const int hkv = d->num_kv_heads, g = d->num_q_heads / hkv;
  // candidates and chunks are described by runs and row ranges, so the host
  // work is O(tables x segments); the kernels expand them
  std::vector<ScoreTable> tables;
  std::vector<ScoreRun> runs;
  std::vector<ScoreRange> ranges;
  std::vector<int32_t> table_map(static_cast<size_t>(dv.n_tables), -1);
  int64_t max_pages = 0, n_chunks = 0, n_cand = 0;
  for (int r = 0; r < n_req; ++r) {
    const int L = lay->cu_seqlens[r + 1] - lay->cu_seqlens[r];
    max_pages = std::max<int64_t>(max_pages, (L + P - 1) / P);
    // the request's rows for retrieval heads: its uncached positions, merged
    const int32_t range_begin = static_cast<int32_t>(ranges.size());
    int last_row = -1, n_rows = 0, req_chunks = 0;
    for (int s = dv.seg_indptr[r]; s < dv.seg_indptr[r + 1]; ++s) {
      const rk_segment& sg = lay->segments[s];
      if (sg.cached || sg.len == 0) continue;
      const int a = sg.logical_start, b = a + sg.len;
      if (static_cast<int32_t>(ranges.size()) > range_begin && ranges.back().end == a) ranges.back().end = b;
      else ranges.push_back(ScoreRange{a, b});
      last_row = b - 1;
      n_rows += sg.len;
    }
    const int32_t range_end = static_cast<int32_t>(ranges.size());
    for (int32_t x = range_begin; x < range_end; ++x)
      req_chunks += (ranges[x].end - ranges[x].begin + kScoreChunkRows - 1) / kScoreChunkRows;
    for (int layer = 0; layer < d->n_layers; ++layer)
      for (int kvh = 0; kvh < hkv; ++kvh) {
        const int lh = layer * hkv + kvh;
        if (lay->class_map[lh] != RK_RETRIEVAL || n_rows == 0) continue;
        const int t = (r * d->n_layers + layer) * hkv + kvh;
        ScoreTable st{};
        st.table = t;
        st.q_row0 = layer * d->total_tokens + lay->cu_seqlens[r];
        st.head0 = kvh * g;
        st.n_rows = n_rows;
        st.range_begin = range_begin;
        st.range_end = range_end;
        st.req_len = L;
        st.chunk_begin = static_cast<int32_t>(n_chunks);
        n_chunks += req_chunks;
        st.chunk_end = static_cast<int32_t>(n_chunks);
        st.cand_begin = static_cast<int32_t>(n_cand);
        st.run_begin = static_cast<int32_t>(runs.size());
        for (int s = dv.seg_indptr[r]; s < dv.seg_indptr[r + 1]; ++s) {
          const rk_segment& sg = lay->segments[s];
          if (!sg.cached || sg.logical_start > last_row) continue;
          const int32_t base = lay->page_base[static_cast<int64_t>(s) * dv.n_lh + lh];
          const int32_t delta = sg.logical_start - sg.stored_pos_base;
          // pages of the segment that start at or before the last row
          const int last_pos = std::min(sg.logical_start + sg.len - 1, last_row);
          const int cnt = (last_pos - sg.logical_start) / P + 1;
          runs.push_back(ScoreRun{static_cast<int32_t>(n_cand), static_cast<int32_t>(n_cand + cnt),
                                  delta, sg.logical_start / P, base, L, {0, 0}});
          n_cand += cnt;
        }
        st.cand_end = static_cast<int32_t>(n_cand);
        st.run_end = static_cast<int32_t>(runs.size());
        if (st.cand_end - st.cand_begin > kScoreMaxCand) return RK_ERR_CAPACITY;
        table_map[static_cast<size_t>(t)] = static_cast<int32_t>(tables.size());
        tables.push_back(st);
      }
  }
  if (n_cand >= kMaxI32 / 8 || n_chunks >= kMaxI32 / 8) return RK_ERR_INVALID_ARG;
  ScoreView& v = out->sv;
  v.n_st = static_cast<int32_t>(tables.size());
  v.n_chunks = static_cast<int32_t>(n_chunks);
  v.n_cand = static_cast<int32_t>(n_cand);
  v.n_runs = static_cast<int32_t>(runs.size());
  v.n_page_blocks = static_cast<int32_t>((n_cand + kScorePagesPerCta - 1) / kScorePagesPerCta);
  v.n_tables = static_cast<int32_t>(dv.n_tables);
  v.top_k = top_k;
  v.hq = d->num_q_heads;
  v.g = g;
  v.n_ranges = static_cast<int32_t>(ranges.size());
  // every array starts on a 16-byte boundary
  auto al4 = [](int32_t w) { return (w + 3) & ~3; };
  int32_t off = al4(static_cast<int32_t>((sizeof(ScoreView) + 3) / 4));
  v.off_tables = off;
  off = al4(off + static_cast<int32_t>(tables.size() * sizeof(ScoreTable) / 4));
  v.off_runs = off;
  off = al4(off + static_cast<int32_t>(runs.size() * sizeof(ScoreRun) / 4));
  v.off_ranges = off;
  off = al4(off + static_cast<int32_t>(ranges.size() * sizeof(ScoreRange) / 4));
  v.off_table_map = off;
  off = al4(off + static_cast<int32_t>(table_map.size()));
  v.off_done = off;
  off = al4(off + static_cast<int32_t>(tables.size()));
  v.off_chunk_table = off;
  off = al4(off + v.n_chunks);
  v.off_block_run = off;
  off = al4(off + v.n_page_blocks);
  v.words = off;
  out->img.assign(static_cast<size_t>(off), 0);
  int32_t* w = out->img.data();
  std::memcpy(w, &v, sizeof v);
  if (!tables.empty()) std::memcpy(w + v.off_tables, tables.data(), tables.size() * sizeof(ScoreTable));
  if (!runs.empty()) std::memcpy(w + v.off_runs, runs.data(), runs.size() * sizeof(ScoreRun));
  if (!ranges.empty()) std::memcpy(w + v.off_ranges, ranges.data(), ranges.size() * sizeof(ScoreRange));
  if (!table_map.empty()) std::memcpy(w + v.off_table_map, table_map.data(), table_map.size() * 4);
  // the lookups the kernels would otherwise search for: a chunk's table and
  // the run holding a page block's first candidate (runs are never empty)
  for (int32_t i = 0; i < v.n_st; ++i)
    for (int32_t c = tables[static_cast<size_t>(i)].chunk_begin; c < tables[static_cast<size_t>(i)].chunk_end; ++c)
      w[v.off_chunk_table + c] = i;
  for (int32_t b = 0, rn = 0; b < v.n_page_blocks; ++b) {
    const int32_t first = b * kScorePagesPerCta;
    while (rn + 1 < v.n_runs && runs[static_cast<size_t>(rn) + 1].cand_begin <= first) ++rn;
    w[v.off_block_run + b] = rn;
  }
  out->max_pages = max_pages;
  out->off_partials = align_up(4 * static_cast<size_t>(off), 256);
  out->off_kbar = align_up(out->off_partials + 4 * static_cast<size_t>(n_chunks) * D, 256);
  // kbar: the scores (4 bytes each), then the rank keys (8 bytes each)
  out->off_urot = align_up(out->off_kbar + 4 * static_cast<size_t>(n_cand + 1) + 8 * static_cast<size_t>(n_cand), 256);
  out->total = align_up(out->off_urot + 4 * runs.size() * D, 256);
  return RK_OK;
}

}  // namespace
}  // namespace rk

using namespace rk;

extern "C" rk_status rk_query_sizes(const rk_dims* dims, const rk_layout* layout, rk_sizes* out) {
  if (!out) return RK_ERR_INVALID_ARG;
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  out->n_tables = dv.n_tables;
  out->entry_capacity = dv.entry_capacity;
  out->range_capacity = dv.range_capacity;
  out->item_capacity = dv.item_capacity;
  out->workspace_bytes = static_cast<int64_t>(dv.map.total);
  return RK_OK;
}

extern "C" rk_status rk_select_visible(const rk_dims* dims, const rk_layout* layout,
                                       const rk_visible* out, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  if (!out || !workspace || !out->entries || !out->entry_start || !out->entry_count ||
      !out->ranges || !out->range_start || !out->range_count)
    return RK_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(out->entries, 16) || !aligned(out->ranges, 8) ||
      !aligned(out->entry_start, 4) || !aligned(out->entry_count, 4) ||
      !aligned(out->range_start, 4) || !aligned(out->range_count, 4))
    return RK_ERR_INVALID_ARG;
  if (out->entry_capacity < dv.entry_capacity || out->range_capacity < dv.range_capacity ||
      workspace_bytes < dv.map.total)
    return RK_ERR_CAPACITY;
  // one host-to-device copy: the layout image (its error word and completion
  // counter zeroed); the select kernel's last CTA rewrites the header
  std::vector<int32_t> img;
  build_layout_image(dims, layout, dv, &img);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemcpyAsync(ws + dv.map.layout, img.data(), 4 * img.size(), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return RK_ERR_CUDA;
  cudaError_t e = launch_select(reinterpret_cast<LayoutView*>(ws + dv.map.layout),
                                static_cast<int>(dv.n_tables), *out,
                                reinterpret_cast<WsHeader*>(ws),
                                reinterpret_cast<Item*>(ws + dv.map.items_tmp),
                                reinterpret_cast<Item*>(ws + dv.map.items),
                                reinterpret_cast<int32_t*>(ws + dv.map.cursor),
                                img[reinterpret_cast<const LayoutView*>(img.data())->off_tile_prefix +
                                    dv.n_tables],
                                s);
  return e == cudaSuccess ? RK_OK : RK_ERR_CUDA;
}

extern "C" rk_status rk_relocate_rope(const void* k_src, int64_t n_src_pages, void* k_dst,
                                      int64_t n_dst_pages, const int32_t* jobs, int32_t n_jobs,
                                      int32_t page_size, int32_t head_dim, double rope_theta,
                                      int32_t* device_error, void* stream) {
  if (n_jobs < 0 || n_src_pages < 1 || n_dst_pages < 1 || page_size < 1 ||
      (head_dim != 64 && head_dim != 128))
    return RK_ERR_INVALID_ARG;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return RK_ERR_INVALID_ARG;
  if (n_jobs > 0 && (!k_src || !k_dst || !jobs)) return RK_ERR_INVALID_ARG;
  if (!aligned(k_src, 16) || !aligned(k_dst, 16) || !aligned(jobs, 4) ||
      !aligned(device_error, 4))
    return RK_ERR_INVALID_ARG;
  cudaError_t e = launch_relocate(k_src, k_dst, jobs, n_jobs, n_src_pages, n_dst_pages,
                                  page_size, head_dim, rope_theta, device_error,
                                  static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RK_OK : RK_ERR_CUDA;
}

extern "C" rk_status rk_segpaged_prefill(const rk_dims* dims, const void* q, const void* k_pool,
                                         const void* v_pool, const rk_visible* vis,
                                         int32_t fuse_rope, double rope_theta, float softmax_scale,
                                         void* o, float* lse, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  if (!q || !k_pool || !v_pool || !vis || !vis->entries || !o || !workspace)
    return RK_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(o, 16) ||
      !aligned(vis->entries, 16) || !aligned(workspace, 256) || !aligned(lse, 4))
    return RK_ERR_INVALID_ARG;
  if (fuse_rope != 0 && fuse_rope != 1) return RK_ERR_INVALID_ARG;
  if (fuse_rope == 1 && (!(rope_theta > 0.0) || !std::isfinite(rope_theta)))
    return RK_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return RK_ERR_INVALID_ARG;
  if (workspace_bytes < sizeof(WsHeader)) return RK_ERR_CAPACITY;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  PrefillLaunchArgs a;
  a.q = q;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.n_layers = dims->n_layers;
  a.hq = dims->num_q_heads;
  a.d = dims->head_dim;
  a.p = dims->page_size;
  a.n_pages = dims->n_pages;
  a.total_tokens = dims->total_tokens;
  a.items = reinterpret_cast<const Item*>(ws + sizeof(WsHeader));
  a.n_items = &hdr->n_items;
  a.work_next = &hdr->work_next;
  a.work_done = &hdr->work_done;
  a.error_word = &hdr->error;
  a.timeout_site = &hdr->timeout_site;
  a.entries = vis->entries;
  a.o = o;
  a.lse = lse;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.fuse_rope = fuse_rope;
  a.rope_theta = rope_theta;
  if (dims->total_tokens == 0) return RK_OK;
  cudaError_t e = launch_prefill_args(a, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? RK_OK : RK_ERR_CUDA;
}

extern "C" rk_status rk_selftest_bounded_wait(int32_t* device_word, int32_t wait_ms,
                                              void* stream) {
  if (!device_word || !aligned(device_word, 4) || wait_ms < 1 || wait_ms > 1000)
    return RK_ERR_INVALID_ARG;
  return launch_selftest_wait(device_word, wait_ms, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? RK_OK
             : RK_ERR_CUDA;
}

extern "C" rk_status rk_get_device_status(const void* workspace, int32_t* status, void* stream) {
  if (!workspace || !status) return RK_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return RK_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, workspace, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess)
    return RK_ERR_CUDA;
  *status = v;
  return v == 0 ? RK_OK : RK_ERR_DEVICE;
}

// ----------------------------------------------------------------------------
// rk_select_visible_noalloc: the page-table stage of rk_select_visible for
// callers that cannot allocate device memory.  Its scratch (the device copy
// of the layout and the device error word) lives in this file-scope array,
// which every GPU that loads the library keeps until the process exits.
// ----------------------------------------------------------------------------

static constexpr size_t kNoAllocScratchBytes = size_t(1) << 20;  // 1 MiB
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name only stands for the symbol, so its address is looked up
// once per device, with that device current, and cached.
rk_status noalloc_scratch_address(uint8_t** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
    return RK_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return RK_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = static_cast<uint8_t*>(g_noalloc_addr[dev]);
  return RK_OK;
}
}  // namespace

extern "C" rk_status rk_select_visible_noalloc(const rk_dims* dims, const rk_layout* layout,
                                               const rk_visible* out, int32_t* device_error,
                                               void* stream) {
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  if (!out || !out->entries || !out->entry_start || !out->entry_count || !out->ranges ||
      !out->range_start || !out->range_count)
    return RK_ERR_INVALID_ARG;
  if (!aligned(out->entries, 16) || !aligned(out->ranges, 8) || !aligned(out->entry_start, 4) ||
      !aligned(out->entry_count, 4) || !aligned(out->range_start, 4) ||
      !aligned(out->range_count, 4) || !aligned(device_error, 4))
    return RK_ERR_INVALID_ARG;
  if (out->entry_capacity < dv.entry_capacity || out->range_capacity < dv.range_capacity)
    return RK_ERR_CAPACITY;
  std::vector<int32_t> img;
  build_layout_image(dims, layout, dv, &img);
  const size_t layout_off = sizeof(WsHeader);
  if (layout_off + 4 * img.size() > kNoAllocScratchBytes) return RK_ERR_CAPACITY;
  uint8_t* scratch = nullptr;
  if ((st = noalloc_scratch_address(&scratch)) != RK_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the scratch keeps the previous call's contents: the header (with the
  // error word) is rewritten as zeros and the layout image is rewritten whole
  WsHeader hdr{};
  hdr.n_tables = static_cast<int32_t>(dv.n_tables);
  if (cudaMemcpyAsync(scratch, &hdr, sizeof hdr, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return RK_ERR_CUDA;
  if (cudaMemcpyAsync(scratch + layout_off, img.data(), 4 * img.size(), cudaMemcpyHostToDevice,
                      s) != cudaSuccess)
    return RK_ERR_CUDA;
  if (launch_select_tables_only(reinterpret_cast<LayoutView*>(scratch + layout_off),
                                static_cast<int>(dv.n_tables), *out,
                                reinterpret_cast<WsHeader*>(scratch), s) != cudaSuccess)
    return RK_ERR_CUDA;
  if (device_error && cudaMemcpyAsync(device_error, scratch, sizeof(int32_t),
                                      cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return RK_ERR_CUDA;
  return RK_OK;
}

extern "C" rk_status rk_score_query_sizes(const rk_dims* dims, const rk_layout* layout,
                                          int32_t top_k, rk_score_sizes* out) {
  if (!out || top_k < 1 || top_k > kScoreMaxTopK) return RK_ERR_INVALID_ARG;
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  if (!layout) return RK_ERR_INVALID_ARG;
  ScoreLayout sl;
  score_layout(dims, layout, &sl);
  Derived dv;
  if ((st = check_layout(dims, &sl.lay, &dv)) != RK_OK) return st;
  ScorePlan plan;
  if ((st = build_score_plan(dims, &sl.lay, dv, top_k, &plan)) != RK_OK) return st;
  out->n_tables = dv.n_tables;
  out->max_pages = plan.max_pages;
  out->workspace_bytes = static_cast<int64_t>(plan.total);
  return RK_OK;
}

extern "C" rk_status rk_score_retrieval_pages(const rk_dims* dims, const rk_layout* layout,
                                              const void* q, const void* k_store, double rope_theta,
                                              int32_t top_k, int32_t* out_pages,
                                              int32_t* out_count, float* out_scores,
                                              int64_t scores_stride, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  if (top_k < 1 || top_k > kScoreMaxTopK) return RK_ERR_INVALID_ARG;
  if (!(rope_theta > 0.0) || !std::isfinite(rope_theta)) return RK_ERR_INVALID_ARG;
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  if (!layout) return RK_ERR_INVALID_ARG;
  ScoreLayout sl;
  score_layout(dims, layout, &sl);
  Derived dv;
  if ((st = check_layout(dims, &sl.lay, &dv)) != RK_OK) return st;
  ScorePlan plan;
  if ((st = build_score_plan(dims, &sl.lay, dv, top_k, &plan)) != RK_OK) return st;
  if (!q || !k_store || !out_pages || !out_count || !workspace) return RK_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_store, 16) || !aligned(out_pages, 4) ||
      !aligned(out_count, 4) || !aligned(out_scores, 4) || !aligned(workspace, 256))
    return RK_ERR_INVALID_ARG;
  if (out_scores && scores_stride < plan.max_pages) return RK_ERR_CAPACITY;
  if (workspace_bytes < plan.total) return RK_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemcpyAsync(ws, plan.img.data(), 4 * plan.img.size(), cudaMemcpyHostToDevice, s) !=
      cudaSuccess)
    return RK_ERR_CUDA;
  double inv_freq[64];
  for (int m = 0; m < dims->head_dim / 2; ++m)
    inv_freq[m] = std::pow(rope_theta, -2.0 * m / dims->head_dim);
  cudaError_t e = launch_score(reinterpret_cast<const ScoreView*>(ws), plan.sv, q, k_store,
                               dims->head_dim, dims->page_size, inv_freq,
                               reinterpret_cast<float*>(ws + plan.off_partials),
                               reinterpret_cast<float*>(ws + plan.off_kbar),
                               reinterpret_cast<float*>(ws + plan.off_urot), out_pages,
                               out_count, out_scores, out_scores ? scores_stride : 0, s);
  return e == cudaSuccess ? RK_OK : RK_ERR_CUDA;
}

// ---- paged decode

namespace rk {
namespace {
void importance_table_pages(const rk_dims* d, const rk_layout* lay, const Derived& dv, int r,
                            int lh, int64_t t, std::vector<int>* out);

struct DecodePlan {
  int64_t n_pieces = 0;
  int n_cta = 0, per = 0;
  int64_t total = 0;                // decode pages of all tables
  std::vector<int32_t> upload;      // req_len [n_req], then DecodeTable [n_tables]
  size_t off_req_len = 0, off_tables = 0, off_part_o = 0, off_part_ml = 0, bytes = 0;
};

// The decode row of request r is its last position.  A table reads the
// entries of its page table (importance_table_pages: the class rule of the
// select kernel) from the first whose last key is at or after the row's
// first visible key; a table whose row set does not hold the row reads
// nothing.  The tables' decode pages, concatenated, are cut into n_cta
// equal ranges, one per CTA (2 per SM), so every CTA streams the same
// number of pages; a range that spans tables gives one partial result per
// (table, CTA) piece.
rk_status plan_decode(const rk_dims* d, const rk_layout* lay, const Derived& dv, DecodePlan* out) {
  const int g = d->num_q_heads / d->num_kv_heads;
  if (g > kDecodeMaxG || dv.n_lh > kDecodeMaxLh) return RK_ERR_INVALID_ARG;
  const int P = d->page_size, hkv = d->num_kv_heads, W = lay->class_window[RK_LOCAL];
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    sms = 148;  // sizes only: the launch queries the device again
  cudaGetLastError();
  const size_t nt = static_cast<size_t>(dv.n_tables);
  std::vector<DecodeTable> tabs(nt);
  std::vector<int> pages;
  int64_t total = 0;
  for (int r = 0; r < d->n_req; ++r) {
    const int L = lay->cu_seqlens[r + 1] - lay->cu_seqlens[r];
    const int row = L - 1;
    bool last_unc = false;  // the request's last position is uncached
    if (L > 0)
      for (int s = dv.seg_indptr[r]; s < dv.seg_indptr[r + 1]; ++s)
        if (lay->segments[s].logical_start + lay->segments[s].len == L) last_unc = !lay->segments[s].cached;
    for (int layer = 0; layer < d->n_layers; ++layer)
      for (int kvh = 0; kvh < hkv; ++kvh) {
        const int lh = layer * hkv + kvh;
        const int64_t t = (static_cast<int64_t>(r) * d->n_layers + layer) * hkv + kvh;
        DecodeTable& dt = tabs[static_cast<size_t>(t)];
        dt.g0 = static_cast<int32_t>(total);
        const int cls = lay->class_map[lh];
        const bool has_row = L > 0 && (cls == RK_GLOBAL || cls == RK_DENSE || last_unc);
        importance_table_pages(d, lay, dv, r, lh, t, &pages);
        dt.n_e = static_cast<int32_t>(pages.size());
        if (!has_row || pages.empty()) continue;
        const int lo = cls == RK_LOCAL ? row - W + 1 : 0;
        int first = 0;
        while (first < dt.n_e && pages[first] + std::min(P, L - pages[first]) - 1 < lo) ++first;
        dt.first = first;
        dt.n_dec = dt.n_e - first;
        total += dt.n_dec;
      }
  }
  if (total >= kMaxI32) return RK_ERR_INVALID_ARG;
  out->total = total;
  out->n_cta = static_cast<int>(std::max<int64_t>(1, std::min<int64_t>(2 * sms, total)));
  out->per = static_cast<int>(std::max<int64_t>(1, (total + out->n_cta - 1) / out->n_cta));
  out->n_cta = static_cast<int>(std::max<int64_t>(1, (total + out->per - 1) / out->per));
  int64_t pieces = 0;
  for (DecodeTable& dt : tabs) {
    dt.piece_base = static_cast<int32_t>(pieces);
    if (dt.n_dec == 0) continue;
    dt.c_first = dt.g0 / out->per;
    dt.n_pieces = (dt.g0 + dt.n_dec - 1) / out->per - dt.c_first + 1;
    pieces += dt.n_pieces;
  }
  out->n_pieces = pieces;
  const int n_req = d->n_req;
  const size_t rl_words = align_up(static_cast<size_t>(n_req), 4);
  out->upload.assign(rl_words + nt * (sizeof(DecodeTable) / 4), 0);
  for (int r = 0; r < n_req; ++r) out->upload[r] = lay->cu_seqlens[r + 1] - lay->cu_seqlens[r];
  std::memcpy(out->upload.data() + rl_words, tabs.data(), nt * sizeof(DecodeTable));
  // the first 256 bytes hold the device error word, then the upload, then
  // one partial (o [G][D], (m, l) [G]) per piece
  out->off_req_len = 256;
  out->off_tables = out->off_req_len + 4 * rl_words;
  out->off_part_o = align_up(out->off_req_len + 4 * out->upload.size(), 256);
  out->off_part_ml = align_up(out->off_part_o + 4 * static_cast<size_t>(pieces) * g * d->head_dim, 256);
  out->bytes = align_up(out->off_part_ml + 8 * static_cast<size_t>(pieces) * g, 256);
  return RK_OK;
}
}  // namespace
}  // namespace rk

extern "C" rk_status rk_decode_query_sizes(const rk_dims* dims, const rk_layout* layout,
                                           rk_decode_sizes* out) {
  if (!out) return RK_ERR_INVALID_ARG;
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  DecodePlan plan;
  if ((st = plan_decode(dims, layout, dv, &plan)) != RK_OK) return st;
  out->n_pieces = plan.n_pieces;
  out->workspace_bytes = static_cast<int64_t>(plan.bytes);
  return RK_OK;
}

extern "C" rk_status rk_segpaged_decode(const rk_dims* dims, const rk_layout* layout,
                                        const void* q, const void* k_pool, const void* v_pool,
                                        const rk_visible* vis, float softmax_scale, void* o,
                                        float* lse, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  DecodePlan plan;
  if ((st = plan_decode(dims, layout, dv, &plan)) != RK_OK) return st;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale)) return RK_ERR_INVALID_ARG;
  if (!q || !k_pool || !v_pool || !vis || !o || !workspace || !vis->entries ||
      !vis->entry_start || !vis->entry_count || !vis->ranges || !vis->range_start ||
      !vis->range_count)
    return RK_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) || !aligned(o, 16) ||
      !aligned(lse, 4) || !aligned(workspace, 256) || !aligned(vis->entries, 16))
    return RK_ERR_INVALID_ARG;
  if (vis->entry_capacity < dv.entry_capacity || vis->range_capacity < dv.range_capacity)
    return RK_ERR_CAPACITY;
  if (workspace_bytes < plan.bytes) return RK_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess ||
      cudaMemcpyAsync(ws + plan.off_req_len, plan.upload.data(), 4 * plan.upload.size(),
                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return RK_ERR_CUDA;
  DecodeLaunchArgs a{};
  a.q = q;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.entries = vis->entries;
  a.entry_start = vis->entry_start;
  a.entry_count = vis->entry_count;
  a.ranges = vis->ranges;
  a.range_start = vis->range_start;
  a.range_count = vis->range_count;
  a.req_len = reinterpret_cast<const int32_t*>(ws + plan.off_req_len);
  a.tables = reinterpret_cast<const DecodeTable*>(ws + plan.off_tables);
  a.o = o;
  a.lse = lse;
  a.part_o = reinterpret_cast<float*>(ws + plan.off_part_o);
  a.part_ml = reinterpret_cast<float*>(ws + plan.off_part_ml);
  a.n_pages = dims->n_pages;
  a.n_req = dims->n_req;
  a.n_layers = dims->n_layers;
  a.hq = dims->num_q_heads;
  a.hkv = dims->num_kv_heads;
  a.d = dims->head_dim;
  a.p = dims->page_size;
  a.n_cta = plan.n_cta;
  a.per = plan.per;
  a.total = static_cast<int>(plan.total);
  a.window = layout->class_window[RK_LOCAL];
  a.softmax_scale = softmax_scale;
  a.cls = layout->class_map;
  a.error_word = reinterpret_cast<int32_t*>(ws);
  return launch_decode(a, s) == cudaSuccess ? RK_OK : RK_ERR_CUDA;
}

// ---- attention importance (sparse FFN token selection)

namespace rk {
namespace {
// Host plan of one rk_attention_importance call.  The work items of a table
// are (256-key block, row chunk) pairs: the key block's entries come from the
// table's page table, which follows the class rule of the select kernel and
// is therefore known here from the layout alone; the row chunk is one of
// kImpChunkCols / G rows that holds a row able to see a key of the block.
// The plan kernel rebuilds the same items from the device page tables and
// checks the count of every table against tplan.
struct ImportancePlan {
  int64_t n_items = 0;
  int max_kb = 0, max_chunks = 0, max_pages = 0;
  std::vector<int32_t> upload;  // cu [n_req + 1], padding, tplan [n_tables] (offset, items)
  size_t off_cu = 0, off_tplan = 0, off_kbinfo = 0, off_chunkinfo = 0, off_inv = 0;
  size_t off_items = 0, off_part = 0, total = 0;
};

// Request-logical page starts of table t's entries (ascending), by the rule
// rk_select_visible applies: every page for global / dense heads; for local
// heads the pages holding a key of some uncached segment's window
// [a - W + 1, b - 1]; for retrieval heads the uncached pages and the listed
// cached pages that start at or before the last uncached position.
void importance_table_pages(const rk_dims* d, const rk_layout* lay, const Derived& dv, int r,
                            int lh, int64_t t, std::vector<int>* out) {
  out->clear();
  const int P = d->page_size, L = lay->cu_seqlens[r + 1] - lay->cu_seqlens[r];
  const int cls = lay->class_map[lh];
  const int W = lay->class_window[RK_LOCAL];
  const int s0 = dv.seg_indptr[r], s1 = dv.seg_indptr[r + 1];
  int last_unc = -1;
  for (int s = s0; s < s1; ++s)
    if (!lay->segments[s].cached)
      last_unc = std::max(last_unc, lay->segments[s].logical_start + lay->segments[s].len - 1);
  std::vector<int> listed;
  if (cls == RK_RETRIEVAL && lay->retr_indptr)
    listed.assign(lay->retr_pages + lay->retr_indptr[t], lay->retr_pages + lay->retr_indptr[t + 1]);
  std::sort(listed.begin(), listed.end());
  for (int s = s0; s < s1; ++s) {
    const rk_segment& g = lay->segments[s];
    for (int pos = g.logical_start; pos < g.logical_start + g.len; pos += P) {
      const int nv = std::min(P, L - pos);
      bool flag = false;
      if (cls == RK_GLOBAL || cls == RK_DENSE) {
        flag = true;
      } else if (cls == RK_LOCAL) {
        for (int u = s0; u < s1 && !flag; ++u) {
          const rk_segment& x = lay->segments[u];
          if (x.cached) continue;
          flag = std::max(pos, x.logical_start - W + 1) <=
                 std::min(pos + nv - 1, x.logical_start + x.len - 1);
        }
      } else {
        flag = !g.cached ||
               (pos <= last_unc && std::binary_search(listed.begin(), listed.end(), pos / P));
      }
      if (flag) out->push_back(pos);
    }
  }
}

rk_status plan_importance(const rk_dims* d, const rk_layout* lay, const Derived& dv,
                          ImportancePlan* out) {
  const int g = d->num_q_heads / d->num_kv_heads;
  if (g > kImpMaxG || dv.n_lh > kImpMaxLh) return RK_ERR_INVALID_ARG;
  const int P = d->page_size, EPK = kImpKeysPerBlock / P, RPC = kImpChunkCols / g;
  const int n_req = d->n_req, hkv = d->num_kv_heads;
  std::vector<int64_t> items(static_cast<size_t>(dv.n_tables), 0);
  std::vector<int> pages;
  std::vector<std::pair<int, int>> rows;
  int max_kb = 0, max_chunks = 0, max_pages = 0;
  for (int r = 0; r < n_req; ++r) {
    const int L = lay->cu_seqlens[r + 1] - lay->cu_seqlens[r];
    max_pages = std::max(max_pages, (L + P - 1) / P);
    max_chunks = std::max(max_chunks, (L + RPC - 1) / RPC);
    std::vector<std::pair<int, int>> unc;  // merged uncached ranges
    for (int s = dv.seg_indptr[r]; s < dv.seg_indptr[r + 1]; ++s) {
      const rk_segment& x = lay->segments[s];
      if (x.cached) continue;
      if (!unc.empty() && unc.back().second == x.logical_start) unc.back().second += x.len;
      else unc.emplace_back(x.logical_start, x.logical_start + x.len);
    }
    for (int layer = 0; layer < d->n_layers; ++layer)
      for (int kvh = 0; kvh < hkv; ++kvh) {
        const int lh = layer * hkv + kvh;
        const int64_t t = (static_cast<int64_t>(r) * d->n_layers + layer) * hkv + kvh;
        const int cls = lay->class_map[lh];
        const bool local = cls == RK_LOCAL;
        rows.clear();
        if (cls == RK_GLOBAL || cls == RK_DENSE) {
          if (L > 0) rows.emplace_back(0, L);
        } else {
          rows = unc;
        }
        if (rows.empty()) continue;
        importance_table_pages(d, lay, dv, r, lh, t, &pages);
        const int n_e = static_cast<int>(pages.size());
        const int n_kb = (n_e + EPK - 1) / EPK;
        max_kb = std::max(max_kb, n_kb);
        int64_t cnt = 0;
        for (int kb = 0; kb < n_kb; ++kb) {
          const int e0 = kb * EPK, e1 = std::min(n_e, e0 + EPK);
          const int pos_lo = pages[e0];
          const int pos_hi = pages[e1 - 1] + std::min(P, L - pages[e1 - 1]) - 1;
          const int hi = local ? std::min(L - 1, pos_hi + lay->class_window[RK_LOCAL] - 1) : L - 1;
          int f = -1, l = -1;
          for (const auto& x : rows)
            if (x.second > pos_lo) { f = std::max(x.first, pos_lo); break; }
          for (auto it = rows.rbegin(); it != rows.rend(); ++it)
            if (it->first <= hi) { l = std::min(it->second - 1, hi); break; }
          if (f >= 0 && l >= 0) cnt += std::max(0, l / RPC - f / RPC + 1);
        }
        items[static_cast<size_t>(t)] = cnt;
      }
  }
  // the work list: tables with more items first (a longest-first order at
  // table granularity), each table's items contiguous
  std::vector<int64_t> order(static_cast<size_t>(dv.n_tables));
  for (int64_t t = 0; t < dv.n_tables; ++t) order[static_cast<size_t>(t)] = t;
  std::stable_sort(order.begin(), order.end(),
                   [&](int64_t x, int64_t y) { return items[x] > items[y]; });
  std::vector<int64_t> off(static_cast<size_t>(dv.n_tables), 0);
  int64_t acc = 0;
  for (int64_t t : order) {
    off[static_cast<size_t>(t)] = acc;
    acc += items[static_cast<size_t>(t)];
  }
  if (acc >= kMaxI32 / kImpKeysPerBlock) return RK_ERR_CAPACITY;
  out->n_items = acc;
  out->max_kb = std::max(max_kb, 1);
  out->max_chunks = std::max(max_chunks, 1);
  out->max_pages = std::max(max_pages, 1);
  const size_t cu_words = align_up(static_cast<size_t>(n_req + 1), 2);
  out->upload.assign(cu_words + 2 * static_cast<size_t>(dv.n_tables), 0);
  for (int r = 0; r <= n_req; ++r) out->upload[r] = lay->cu_seqlens[r];
  for (int64_t t = 0; t < dv.n_tables; ++t) {
    out->upload[cu_words + 2 * t] = static_cast<int32_t>(off[static_cast<size_t>(t)]);
    out->upload[cu_words + 2 * t + 1] = static_cast<int32_t>(items[static_cast<size_t>(t)]);
  }
  // workspace: header (error word, timeout site, work counter), the upload,
  // the plan kernel's index arrays, the work list and one partial per item
  const size_t nt = static_cast<size_t>(dv.n_tables);
  out->off_cu = 256;
  out->off_tplan = out->off_cu + 4 * cu_words;
  out->off_kbinfo = align_up(out->off_cu + 4 * out->upload.size(), 256);
  out->off_chunkinfo = align_up(out->off_kbinfo + 8 * nt * out->max_kb, 256);
  out->off_inv = align_up(out->off_chunkinfo + 8 * nt * out->max_chunks, 256);
  out->off_items = align_up(out->off_inv + 4 * nt * out->max_pages, 256);
  out->off_part = align_up(out->off_items + 16 * static_cast<size_t>(acc), 256);
  out->total = align_up(out->off_part + 4 * static_cast<size_t>(kImpKeysPerBlock) * acc, 256);
  return RK_OK;
}
}  // namespace
}  // namespace rk

extern "C" rk_status rk_importance_query_sizes(const rk_dims* dims, const rk_layout* layout,
                                               rk_importance_sizes* out) {
  if (!out) return RK_ERR_INVALID_ARG;
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  ImportancePlan plan;
  if ((st = plan_importance(dims, layout, dv, &plan)) != RK_OK) return st;
  out->n_items = plan.n_items;
  out->workspace_bytes = static_cast<int64_t>(plan.total);
  return RK_OK;
}

extern "C" rk_status rk_attention_importance(const rk_dims* dims, const rk_layout* layout,
                                             const void* q, const void* k_pool,
                                             const rk_visible* vis, const float* lse,
                                             float softmax_scale, int32_t top_k,
                                             float* importance, int32_t* tokens,
                                             int32_t* token_count, void* workspace,
                                             size_t workspace_bytes, void* stream) {
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  ImportancePlan plan;
  if ((st = plan_importance(dims, layout, dv, &plan)) != RK_OK) return st;
  if (!(softmax_scale > 0.f) || !std::isfinite(softmax_scale) || top_k < 0)
    return RK_ERR_INVALID_ARG;
  if (!q || !k_pool || !vis || !lse || !importance || !workspace || !vis->entries ||
      !vis->entry_start || !vis->entry_count || !vis->ranges || !vis->range_start ||
      !vis->range_count)
    return RK_ERR_INVALID_ARG;
  if (top_k > 0 && (!tokens) != (!token_count)) return RK_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k_pool, 16) || !aligned(lse, 4) || !aligned(importance, 4) ||
      !aligned(tokens, 4) || !aligned(token_count, 4) || !aligned(workspace, 256) ||
      !aligned(vis->entries, 16))
    return RK_ERR_INVALID_ARG;
  if (vis->entry_capacity < dv.entry_capacity || vis->range_capacity < dv.range_capacity)
    return RK_ERR_CAPACITY;
  if (workspace_bytes < plan.total) return RK_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess ||
      cudaMemcpyAsync(ws + plan.off_cu, plan.upload.data(), 4 * plan.upload.size(),
                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return RK_ERR_CUDA;
  ImportanceLaunchArgs a{};
  a.q = q;
  a.k_pool = k_pool;
  a.entries = vis->entries;
  a.entry_start = vis->entry_start;
  a.entry_count = vis->entry_count;
  a.ranges = vis->ranges;
  a.range_start = vis->range_start;
  a.range_count = vis->range_count;
  a.cu = reinterpret_cast<const int32_t*>(ws + plan.off_cu);
  a.tplan = reinterpret_cast<const int2*>(ws + plan.off_tplan);
  a.kbinfo = reinterpret_cast<int2*>(ws + plan.off_kbinfo);
  a.chunkinfo = reinterpret_cast<int2*>(ws + plan.off_chunkinfo);
  a.inv = reinterpret_cast<int32_t*>(ws + plan.off_inv);
  a.items = reinterpret_cast<int4*>(ws + plan.off_items);
  a.part = reinterpret_cast<float*>(ws + plan.off_part);
  a.lse = lse;
  a.importance = importance;
  a.tokens = tokens;
  a.token_count = token_count;
  a.work_next = reinterpret_cast<int*>(ws + 8);
  a.timeout_site = reinterpret_cast<int*>(ws + 4);
  a.n_pages = dims->n_pages;
  a.n_req = dims->n_req;
  a.n_layers = dims->n_layers;
  a.hq = dims->num_q_heads;
  a.hkv = dims->num_kv_heads;
  a.d = dims->head_dim;
  a.p = dims->page_size;
  a.total_tokens = dims->total_tokens;
  a.window = layout->class_window[RK_LOCAL];
  a.top_k = top_k;
  a.n_items = static_cast<int>(plan.n_items);
  a.max_kb = plan.max_kb;
  a.max_chunks = plan.max_chunks;
  a.max_pages = plan.max_pages;
  a.softmax_scale = softmax_scale;
  a.cls = layout->class_map;
  a.error_word = reinterpret_cast<int32_t*>(ws);
  return launch_importance(a, s) == cudaSuccess ? RK_OK : RK_ERR_CUDA;
}

// ---- token-selective FFN

namespace rk {
namespace {
struct FfnPlan {
  int64_t m = 0;
  std::vector<int32_t> upload;  // cu [n_req + 1], selection prefix [n_req + 1]
  size_t off_up = 0, off_rows = 0, off_xs = 0, off_h = 0, total = 0;
};
rk_status plan_ffn(const rk_ffn_dims* d, int32_t n_req, const int32_t* cu, int32_t top_k,
                   FfnPlan* out) {
  if (!d || !cu || n_req < 1 || top_k < 0 || d->reserved != 0 || d->n_rows < 0)
    return RK_ERR_INVALID_ARG;
  if (d->d_model < 256 || d->d_model % 256 != 0 || d->d_ff < 128 || d->d_ff % 128 != 0 ||
      d->d_model > (1 << 16) || d->d_ff > (1 << 18))
    return RK_ERR_INVALID_ARG;
  if (cu[0] != 0 || cu[n_req] != d->n_rows) return RK_ERR_INVALID_ARG;
  out->upload.assign(2 * static_cast<size_t>(n_req + 1), 0);
  int64_t m = 0;
  for (int r = 0; r < n_req; ++r) {
    if (cu[r + 1] < cu[r]) return RK_ERR_INVALID_ARG;
    out->upload[r] = cu[r];
    out->upload[n_req + 1 + r] = static_cast<int32_t>(m);
    m += std::min<int64_t>(top_k, cu[r + 1] - cu[r]);
  }
  out->upload[n_req] = cu[n_req];
  out->upload[2 * n_req + 1] = static_cast<int32_t>(m);
  if (m >= kMaxI32 / 2) return RK_ERR_INVALID_ARG;
  out->m = m;
  out->off_up = 256;
  out->off_rows = align_up(out->off_up + 4 * out->upload.size(), 256);
  out->off_xs = align_up(out->off_rows + 4 * static_cast<size_t>(m), 256);
  out->off_h = align_up(out->off_xs + 2 * static_cast<size_t>(m) * d->d_model, 256);
  out->total = align_up(out->off_h + 2 * static_cast<size_t>(m) * d->d_ff, 256);
  return RK_OK;
}
}  // namespace
}  // namespace rk

extern "C" rk_status rk_ffn_query_sizes(const rk_ffn_dims* dims, int32_t n_req,
                                        const int32_t* cu_seqlens, int32_t top_k,
                                        rk_ffn_sizes* out) {
  if (!out) return RK_ERR_INVALID_ARG;
  FfnPlan plan;
  rk_status st = plan_ffn(dims, n_req, cu_seqlens, top_k, &plan);
  if (st != RK_OK) return st;
  out->n_selected = plan.m;
  out->workspace_bytes = static_cast<int64_t>(plan.total);
  return RK_OK;
}

extern "C" rk_status rk_sparse_ffn(const rk_ffn_dims* dims, int32_t n_req,
                                   const int32_t* cu_seqlens, const int32_t* tokens, int32_t top_k,
                                   void* x, const void* w_gate, const void* w_up,
                                   const void* w_down, void* workspace, size_t workspace_bytes,
                                   void* stream) {
  FfnPlan plan;
  rk_status st = plan_ffn(dims, n_req, cu_seqlens, top_k, &plan);
  if (st != RK_OK) return st;
  if (!x || !w_gate || !w_up || !w_down || !workspace || (plan.m > 0 && !tokens))
    return RK_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(w_gate, 16) || !aligned(w_up, 16) || !aligned(w_down, 16) ||
      !aligned(tokens, 4) || !aligned(workspace, 256))
    return RK_ERR_INVALID_ARG;
  if (workspace_bytes < plan.total) return RK_ERR_CAPACITY;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess ||
      cudaMemcpyAsync(ws + plan.off_up, plan.upload.data(), 4 * plan.upload.size(),
                      cudaMemcpyHostToDevice, s) != cudaSuccess)
    return RK_ERR_CUDA;
  FfnLaunchArgs a{};
  a.x = x;
  a.w_gate = w_gate;
  a.w_up = w_up;
  a.w_down = w_down;
  a.cu = reinterpret_cast<const int32_t*>(ws + plan.off_up);
  a.sel_prefix = a.cu + (n_req + 1);
  a.tokens = tokens;
  a.xs = ws + plan.off_xs;
  a.h = ws + plan.off_h;
  a.rows = reinterpret_cast<int32_t*>(ws + plan.off_rows);
  a.error_word = reinterpret_cast<int32_t*>(ws);
  a.timeout_site = reinterpret_cast<int*>(ws + 4);
  a.m = static_cast<int>(plan.m);
  a.n_req = n_req;
  a.top_k = top_k;
  a.d_model = dims->d_model;
  a.d_ff = dims->d_ff;
  return launch_sparse_ffn(a, s) == cudaSuccess ? RK_OK : RK_ERR_CUDA;
}

// ---- relocation plan (the relocate-mode step's job lists)

namespace rk {
namespace {
struct RelocPlan {
  std::vector<int32_t> jobs_k, jobs_v;  // [n][3] (src_page, dst_page, delta)
  std::vector<int32_t> page_base;       // [n_segments][n_lh]
  int64_t n_extra = 0;
};

// Pages attention reads are the page-table entries, which follow from the
// layout by the class rule (importance_table_pages).  Every visible page of
// a cached instance with delta != 0 is rotated into the working pool at its
// own id; a physical page visible through two instances at different
// deltas keeps its id for the first and gets a fresh run of pages appended
// to both pools for the later one (K rotated, V copied).
rk_status plan_relocation(const rk_dims* d, const rk_layout* lay, const Derived& dv,
                          RelocPlan* out) {
  const int P = d->page_size, hkv = d->num_kv_heads;
  const int64_t n_lh = dv.n_lh;
  const int n_seg = lay->n_segments;
  // need[s * n_lh + lh]: page offsets within segment s that a table lists
  std::vector<std::vector<int>> need(static_cast<size_t>(n_seg) * n_lh);
  std::vector<int> pages;
  for (int r = 0; r < d->n_req; ++r) {
    const int s0 = dv.seg_indptr[r], s1 = dv.seg_indptr[r + 1];
    if (s0 == s1) continue;
    for (int layer = 0; layer < d->n_layers; ++layer)
      for (int kvh = 0; kvh < hkv; ++kvh) {
        const int lh = layer * hkv + kvh;
        const int64_t t = (static_cast<int64_t>(r) * d->n_layers + layer) * hkv + kvh;
        importance_table_pages(d, lay, dv, r, lh, t, &pages);
        int s = s0;
        for (int pos : pages) {
          while (s + 1 < s1 && lay->segments[s + 1].logical_start <= pos) ++s;
          need[static_cast<size_t>(s) * n_lh + lh].push_back((pos - lay->segments[s].logical_start) / P);
        }
      }
  }
  out->page_base.assign(lay->page_base, lay->page_base + static_cast<size_t>(n_seg) * n_lh);
  std::vector<int64_t> claim(static_cast<size_t>(d->n_pages), INT64_MIN);  // delta held per page
  int64_t nxt = d->n_pages;
  for (int s = 0; s < n_seg; ++s) {
    const rk_segment& g = lay->segments[s];
    const int delta = g.cached ? g.logical_start - g.stored_pos_base : 0;
    const int npg = (g.len + P - 1) / P;
    for (int64_t lh = 0; lh < n_lh; ++lh) {
      std::vector<int>& ks = need[static_cast<size_t>(s) * n_lh + lh];
      if (ks.empty()) continue;
      std::sort(ks.begin(), ks.end());
      ks.erase(std::unique(ks.begin(), ks.end()), ks.end());
      const int64_t base = lay->page_base[static_cast<size_t>(s) * n_lh + lh];
      bool clash = false;
      for (int k : ks) {
        const int64_t c = claim[static_cast<size_t>(base + k)];
        clash |= c != INT64_MIN && c != delta;
      }
      if (clash) {
        if (nxt + npg >= kMaxI32 / P) return RK_ERR_CAPACITY;
        out->page_base[static_cast<size_t>(s) * n_lh + lh] = static_cast<int32_t>(nxt);
        for (int k : ks) {
          out->jobs_k.insert(out->jobs_k.end(), {static_cast<int32_t>(base + k),
                                                 static_cast<int32_t>(nxt + k), delta});
          out->jobs_v.insert(out->jobs_v.end(), {static_cast<int32_t>(base + k),
                                                 static_cast<int32_t>(nxt + k), 0});
        }
        nxt += npg;
        continue;
      }
      for (int k : ks) {
        int64_t& c = claim[static_cast<size_t>(base + k)];
        if (c != INT64_MIN) continue;
        c = delta;
        if (delta != 0)
          out->jobs_k.insert(out->jobs_k.end(), {static_cast<int32_t>(base + k),
                                                 static_cast<int32_t>(base + k), delta});
      }
    }
  }
  out->n_extra = nxt - d->n_pages;
  return RK_OK;
}
}  // namespace
}  // namespace rk

extern "C" rk_status rk_relocation_query_sizes(const rk_dims* dims, const rk_layout* layout,
                                               rk_relocation_sizes* out) {
  if (!out) return RK_ERR_INVALID_ARG;
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  RelocPlan plan;
  if ((st = plan_relocation(dims, layout, dv, &plan)) != RK_OK) return st;
  out->n_jobs_k = static_cast<int64_t>(plan.jobs_k.size() / 3);
  out->n_jobs_v = static_cast<int64_t>(plan.jobs_v.size() / 3);
  out->n_extra_pages = plan.n_extra;
  return RK_OK;
}

extern "C" rk_status rk_relocation_plan(const rk_dims* dims, const rk_layout* layout,
                                        int32_t* jobs_k, int64_t cap_k, int32_t* jobs_v,
                                        int64_t cap_v, rk_segment* segments_out,
                                        int32_t* page_base_out) {
  rk_status st = check_dims(dims);
  if (st != RK_OK) return st;
  Derived dv;
  if ((st = check_layout(dims, layout, &dv)) != RK_OK) return st;
  if ((layout->n_segments > 0 && (!segments_out || !page_base_out)) || cap_k < 0 || cap_v < 0)
    return RK_ERR_INVALID_ARG;
  RelocPlan plan;
  if ((st = plan_relocation(dims, layout, dv, &plan)) != RK_OK) return st;
  const int64_t nk = static_cast<int64_t>(plan.jobs_k.size() / 3);
  const int64_t nv = static_cast<int64_t>(plan.jobs_v.size() / 3);
  if (nk > cap_k || nv > cap_v) return RK_ERR_CAPACITY;
  if ((nk > 0 && !jobs_k) || (nv > 0 && !jobs_v)) return RK_ERR_INVALID_ARG;
  if (nk > 0) std::memcpy(jobs_k, plan.jobs_k.data(), 4 * plan.jobs_k.size());
  if (nv > 0) std::memcpy(jobs_v, plan.jobs_v.data(), 4 * plan.jobs_v.size());
  for (int s = 0; s < layout->n_segments; ++s) {
    segments_out[s] = layout->segments[s];
    segments_out[s].stored_pos_base = layout->segments[s].logical_start;
  }
  if (layout->n_segments > 0)
    std::memcpy(page_base_out, plan.page_base.data(), 4 * plan.page_base.size());
  return RK_OK;
}
