// Internal layout of the workspace and the work list shared by the
// library's translation units.  Not part of the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/rk.h"

namespace rk {

constexpr int kRowsPerTile = 128;  // query rows per Q tile (one TMEM lane per row)
constexpr int kKeysPerTile = 128;  // keys per KV tile (N of the QK^T MMA)
// Work items are ordered by cost (KV tiles) in this many buckets, longest
// first; costs past the last bucket share it.  With several requests or
// layers the buckets are split between (request, layer) groups, taken one
// group after another, so the items that run side by side read the pages of
// few tables (their K / V stays in L2).
constexpr int kCostBuckets = 2048;
constexpr int kMaxBucketGroups = 256;

// Workspace header (first 256 bytes of the workspace).
struct WsHeader {
  int32_t error;          // RK_DEV_* bits, reset by rk_select_visible
  int32_t n_items;        // attention work items written by the select kernels
  int32_t n_tables;
  int32_t item_capacity;
  int32_t timeout_site;   // first bounded wait that gave up (diagnostics)
  int32_t work_next;      // attention: next work item to hand out (dynamic schedule)
  int32_t work_done;      // attention: CTAs finished (the last one resets both)
  int32_t pad[57];
};
static_assert(sizeof(WsHeader) == 256, "header size");

// One attention work item: up to two q heads of one kv head over the same
// block of <= 128 rows, hence the same visible keys (GQA sharing).
struct Item {
  int32_t q_row0;     // layer * T + first token of the request
  int32_t row_begin;  // request-local rows [row_begin, row_end)
  int32_t row_end;
  int32_t e_begin;    // entries [e_begin, e_end) of the rk_visible arrays
  int32_t e_end;
  int32_t qh0;        // first q head
  int32_t nh;         // 1 or 2 q heads
  int32_t window;     // key window (local class), -1 = unbounded
  int32_t layer;
  int32_t req;
  int32_t table;
  int32_t cost;       // KV tiles
};
static_assert(sizeof(Item) == 48, "item size");

// Layout copy inside the workspace, as written by the host (all int32).
struct LayoutView {
  int32_t n_req, n_layers, hq, hkv, d, p, n_seg, n_retr;
  int64_t n_pages;
  int32_t total_tokens, total_pages;  // total_pages = sum_r ceil(L_r / P)
  int32_t window;                     // class_window[RK_LOCAL]
  int32_t item_capacity;
  int32_t max_table_pages;            // max_r ceil(L_r / P)
  // work-list order: bucket_groups groups of kCostBuckets / bucket_groups
  // cost buckets each (group = request x n_layers + layer when bucket_groups
  // > 1, else one group), longest first inside a group, cost_width KV tiles
  // per bucket
  int32_t bucket_groups;
  int32_t cost_width;
  // written by the select kernel (the host uploads them as zero each call)
  int32_t error;       // RK_DEV_* bits raised while selecting
  int32_t done_count;  // CTAs of the select kernel that finished their table
  // offsets (in int32 elements from the start of the layout block)
  int32_t off_seg;          // [n_seg][5]
  int32_t off_seg_indptr;   // [n_req + 1]
  int32_t off_page_base;    // [n_seg][n_layers * hkv]
  int32_t off_cu;           // [n_req + 1]
  int32_t off_page_prefix;  // [n_req + 1]
  int32_t off_class;        // [n_layers * hkv]
  int32_t off_retr_indptr;  // [n_tables + 1]
  int32_t off_retr_pages;   // [n_retr]
  int32_t off_tile_prefix;  // [n_tables + 1] exclusive prefix of the work items per table
  int32_t off_cost_hist;    // [kCostBuckets] items per cost bucket (uploaded as zero)
  int32_t layout_words;
};

// Workspace map (byte offsets), computed on the host.
struct WsMap {
  size_t header = 0;
  size_t items = 0;      // Item[item_capacity], sorted by cost (longest first)
  size_t items_tmp = 0;  // Item[item_capacity], unsorted
  size_t cursor = 0;     // int32[kCostBuckets]: next sorted slot of each cost bucket
  size_t layout = 0;     // LayoutView followed by the int32 arrays
  size_t total = 0;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Arguments of one attention launch (device pointers).
struct PrefillLaunchArgs {
  const void* q;
  const void* k_pool;
  const void* v_pool;
  int n_layers, hq, d, p;
  int64_t n_pages;
  int total_tokens;
  const Item* items;
  const int32_t* n_items;
  int* work_next;
  int* work_done;
  int* error_word;
  int* timeout_site;
  const rk_entry* entries;
  void* o;
  float* lse;
  float scale_log2;
  int fuse_rope;
  double rope_theta;
};

// ---- retrieval page scoring (host image read by the scoring kernels)

constexpr int kScoreChunkRows = 64;   // query rows summed by one CTA
constexpr int kScorePagesPerCta = 8;  // candidate pages per CTA (one warp each)
constexpr int kScoreMaxCand = 4096;   // candidate pages of one table
constexpr int kScoreMaxTopK = 64;

struct ScoreTable {  // one retrieval table that has rows
  int32_t table;     // table id
  int32_t q_row0;    // layer * T + cu[r]: packed q row of the request's position 0
  int32_t head0;     // first q head of the kv head
  int32_t n_rows;    // computed rows (uncached positions)
  int32_t chunk_begin, chunk_end;  // its query chunks (kScoreChunkRows rows of one range each)
  int32_t cand_begin, cand_end;    // its candidate pages (ascending page)
  int32_t run_begin, run_end;      // its runs of candidates sharing one delta
  int32_t range_begin, range_end;  // its row ranges (the request's uncached rows, merged)
  int32_t req_len;
  int32_t pad[3];
};
struct ScoreRun {  // candidates [cand_begin, cand_end): consecutive pages of one cached segment
  int32_t cand_begin, cand_end, delta;
  int32_t first_page;  // request page of the run's first candidate
  int32_t phys_base;   // its physical page (the run's pages are consecutive ids)
  int32_t req_len;     // length of the request (keys of its last page)
  int32_t pad[2];
};
struct ScoreRange {  // request-local rows [begin, end)
  int32_t begin, end;
};
struct ScoreView {
  int32_t n_st, n_chunks, n_cand, n_runs, n_page_blocks, n_tables, top_k;
  int32_t hq, g, n_ranges;
  int32_t off_tables;     // ScoreTable[n_st]
  int32_t off_runs;       // ScoreRun[n_runs]
  int32_t off_ranges;     // ScoreRange[n_ranges]
  int32_t off_table_map;  // int32[n_tables]: score table of a table, -1 if none
  int32_t off_done;       // int32[n_st]: query chunks finished per score table (zero when uploaded)
  int32_t off_chunk_table;  // int32[n_chunks]: score table of each query chunk
  int32_t off_block_run;    // int32[n_page_blocks]: run of each page block's first candidate
  int32_t words;
};

// Three launches: query chunk sums (the last chunk of a table forms the
// rotated u of its runs), page scores (key means dotted with their run's
// rotated u), and the picks, one CTA per table.
cudaError_t launch_score(const ScoreView* sv_dev, const ScoreView& sv_host, const void* q,
                         const void* k_store, int D, int P, const double* inv_freq_host,
                         float* partials, float* scores, float* urot, int32_t* out_pages,
                         int32_t* out_count, float* out_scores, int64_t scores_stride,
                         cudaStream_t stream);

// ---- paged decode

constexpr int kDecodeMaxLh = 1024;  // layers x kv heads per call
constexpr int kDecodeMaxG = 8;      // q heads per kv head

struct DecodeTable {  // one table's decode work (host-computed, uploaded)
  int32_t g0;          // its first page in the concatenated decode pages of all tables
  int32_t first;       // its first decode entry (page-table index)
  int32_t n_dec;       // decode entries (0: the table reads nothing)
  int32_t n_e;         // page-table entries the host expects (checked on the device)
  int32_t piece_base;  // its first partial result
  int32_t c_first;     // the CTA of its first piece
  int32_t n_pieces;    // pieces (consecutive CTAs)
  int32_t pad;
};

struct DecodeLaunchArgs {
  const void* q;  // bf16 [n_layers][n_req][hq][d]
  const void* k_pool;
  const void* v_pool;
  const rk_entry* entries;
  const int32_t* entry_start;
  const int32_t* entry_count;
  const rk_range* ranges;
  const int32_t* range_start;
  const int32_t* range_count;
  const int32_t* req_len;      // device [n_req]
  const DecodeTable* tables;   // device [n_tables]
  void* o;     // bf16 [n_layers][n_req][hq][d]
  float* lse;  // fp32 [n_layers][hq][n_req] or null
  float* part_o;
  float* part_ml;
  int64_t n_pages;
  int n_req, n_layers, hq, hkv, d, p, n_cta, per, total, window;
  float softmax_scale;
  const int8_t* cls;  // host [n_layers * hkv]
  int32_t* error_word;
};

cudaError_t launch_decode(const DecodeLaunchArgs& a, cudaStream_t stream);

// ---- attention importance (sparse FFN token selection)
constexpr int kImpKeysPerBlock = 256;  // keys of one table per work item (two MMA halves)
constexpr int kImpChunkCols = 4096;    // (row, q head) columns per row chunk: 4096 / G rows
constexpr int kImpMaxLh = 1024;        // layers x kv heads per call
constexpr int kImpMaxG = 8;            // q heads per kv head

struct ImportanceLaunchArgs {
  const void* q;       // bf16 [n_layers][T][hq][d], the prefill's queries
  const void* k_pool;  // bf16 [n_pages][p][d], relocated
  const rk_entry* entries;
  const int32_t* entry_start;
  const int32_t* entry_count;
  const rk_range* ranges;
  const int32_t* range_start;
  const int32_t* range_count;
  const int32_t* cu;     // device [n_req + 1]
  const int2* tplan;     // device [n_tables]: (work-list offset, items) of each table
  int2* kbinfo;          // device [n_tables][max_kb]
  int2* chunkinfo;       // device [n_tables][max_chunks]
  int32_t* inv;          // device [n_tables][max_pages]
  int4* items;           // device [n_items]
  float* part;           // device [n_items][kImpKeysPerBlock]
  const float* lse;      // fp32 [n_layers][hq][T], natural log (the prefill's)
  float* importance;     // fp32 [n_layers][T]
  int32_t* tokens;       // [n_layers][n_req][top_k] or null
  int32_t* token_count;  // [n_layers][n_req] or null
  int* work_next;        // zeroed by the caller
  int* timeout_site;
  int64_t n_pages;
  int n_req, n_layers, hq, hkv, d, p, total_tokens, window, top_k;
  int n_items, max_kb, max_chunks, max_pages;
  float softmax_scale;
  const int8_t* cls;   // host [n_layers * hkv]
  int32_t* error_word;
};

cudaError_t launch_importance(const ImportanceLaunchArgs& a, cudaStream_t stream);

}  // namespace rk

namespace rk {

// ---- token-selective FFN
struct FfnLaunchArgs {
  void* x;                    // bf16 [n_rows][d_model], updated in place
  const void* w_gate;         // bf16 [d_ff][d_model]
  const void* w_up;           // bf16 [d_ff][d_model]
  const void* w_down;         // bf16 [d_model][d_ff]
  const int32_t* cu;          // device [n_req + 1]
  const int32_t* sel_prefix;  // device [n_req + 1]: selection entries before request r
  const int32_t* tokens;      // device [n_req][top_k], request-local
  void* xs;                   // workspace bf16 [m][d_model]
  void* h;                    // workspace bf16 [m][d_ff]
  int32_t* rows;              // workspace [m]
  int32_t* error_word;
  int* timeout_site;
  int m, n_req, top_k, d_model, d_ff;
};

cudaError_t launch_sparse_ffn(const FfnLaunchArgs& a, cudaStream_t stream);

}  // namespace rk
