/*
 * rk.h — C ABI of the SegPagedAttention prefill library (librk.so, sm_100a).
 *
 * The operations follow the RedKnot pages:
 *   - rk_select_visible   <- SELECTVISIBLESTATE (paooo page, "how to use":
 *                            choose which reused KV each head sees), built on
 *                            the per-(layer, kv_head) head class map and the
 *                            "per-head page table + segmented KV store" of the
 *                            README excerpt ("SegPagedAttention Runtime").
 *   - rk_relocate_rope    <- "Offline KV Reuse + RoPE Relocation" (README
 *                            excerpt): re-rotate cached K from the position it
 *                            was stored at to its new absolute position.
 *   - rk_segpaged_prefill <- EXECUTE's attention (paooo page, "how to use" and
 *                            "technical principles": a fused varlen kernel over
 *                            per-head pages that never builds an attn_mask).
 * and, beside the hot path, retrieval page scoring, paged decode, the
 * attention importance and the token-selective FFN it feeds (each section
 * below cites its passage).
 *
 * Conventions shared by every call
 *   - All pointers are caller-owned.  The library never allocates or frees
 *     memory; device buffers are passed in, sized by rk_query_sizes().
 *   - "host" pointers are read during the call only.  "device" pointers must
 *     address memory of the current CUDA device.
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).
 *     Every device-side effect is ordered on that stream; calls return before
 *     the GPU work finishes, except rk_get_device_status().
 *   - Argument errors are detected on the host, synchronously, before any
 *     GPU work is enqueued; nothing is written in that case.
 *   - Kernels never trap.  A fault they detect (a page id outside the pool, a
 *     bounded wait that ran out) sets a bit in the device error word inside
 *     the workspace; read it with rk_get_device_status().
 *   - bf16 tensors are passed as raw 16-bit storage (const void*).
 *
 * Notation: T = total tokens of the batch, L_r = length of request r,
 * Hq / Hkv = query / key-value heads (G = Hq / Hkv, q head h reads kv head
 * h / G), D = head_dim, P = page_size.  A "table" is one
 * (request, layer, kv_head); its index is t = (r * n_layers + layer) * Hkv + kvh.
 */
#ifndef RK_H_
#define RK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t rk_status;
#define RK_OK 0
#define RK_ERR_INVALID_ARG 1 /* null pointer, bad dims, D not in {64,128}, P not in {16,64}, ... */
#define RK_ERR_UNALIGNED 2   /* a segment other than a request's last has len % P != 0 */
#define RK_ERR_CAPACITY 3    /* a buffer or the workspace is smaller than rk_query_sizes() says */
#define RK_ERR_CUDA 4        /* a CUDA runtime / driver call failed */
#define RK_ERR_DEVICE 5      /* rk_get_device_status(): the device error word is non-zero */

/* bits of the device error word (reported through rk_get_device_status) */
#define RK_DEV_BAD_PAGE 1u   /* a page id outside [0, n_pages): the access was skipped */
#define RK_DEV_TIMEOUT 2u    /* a bounded wait inside a kernel gave up: outputs are invalid */
#define RK_DEV_CAPACITY 4u   /* a work list would not fit the workspace: outputs are invalid */

/* head classes (README excerpt, "Head Classification") */
#define RK_GLOBAL 0    /* every row; key j visible to row i iff j <= i */
#define RK_LOCAL 1     /* uncached rows; visible iff i - W < j <= i (W = class_window[RK_LOCAL]) */
#define RK_RETRIEVAL 2 /* uncached rows; visible iff j <= i and (j uncached or page(j) listed) */
#define RK_DENSE 3     /* same visibility as RK_GLOBAL (its KV is recomputed upstream) */

typedef struct {
  int32_t n_req;        /* requests in the batch, >= 1 */
  int32_t n_layers;     /* attention layers covered by one call, >= 1 */
  int32_t num_q_heads;  /* Hq, a multiple of num_kv_heads */
  int32_t num_kv_heads; /* Hkv */
  int32_t head_dim;     /* D: 64 or 128 */
  int32_t page_size;    /* P: 16 or 64 */
  int64_t n_pages;      /* pages in k_pool / v_pool; n_pages * P < 2^31 */
  int32_t total_tokens; /* T = cu_seqlens[n_req] */
  int32_t reserved;     /* must be 0 */
} rk_dims;

/* One segment instance of a request.  Segments of a request are listed in
 * ascending logical_start and tile [0, L_r) exactly.  Cached segments hold KV
 * computed offline at positions stored_pos_base .. stored_pos_base + len - 1
 * and reused here at logical_start (delta = logical_start - stored_pos_base);
 * uncached segments hold KV computed for this request at its own positions
 * (their stored_pos_base is ignored, delta = 0). */
typedef struct {
  int32_t req;
  int32_t logical_start;
  int32_t len;
  int32_t stored_pos_base;
  int32_t cached; /* 1 = reused from the offline store, 0 = computed online */
} rk_segment;

/* Host-side description of the batch (all pointers are host memory). */
typedef struct {
  int32_t n_segments;
  const rk_segment* segments; /* [n_segments], grouped by request */
  /* [n_segments][n_layers * Hkv]: physical page of the segment's first page
   * for (layer, kv_head); its pages for that pair are consecutive ids. */
  const int32_t* page_base;
  const int32_t* cu_seqlens;   /* [n_req + 1], cu_seqlens[0] = 0, non-decreasing */
  const int8_t* class_map;     /* [n_layers * Hkv], RK_GLOBAL .. RK_DENSE */
  const int32_t* class_window; /* [4]; class_window[RK_LOCAL] = W >= 1, others unused */
  /* retrieval page lists, CSR over tables ([n_tables + 1] and the values):
   * request-logical page numbers k (positions [kP, kP + P)); listed pages that
   * are uncached or past the request are ignored.  Both may be NULL when no
   * table has class RK_RETRIEVAL. */
  const int32_t* retr_indptr;
  const int32_t* retr_pages;
} rk_layout;

/* One page-table entry (16 bytes). */
typedef struct {
  int32_t phys_page;   /* page id in the pool */
  int32_t logical_pos; /* absolute position (within the request) of the page's first key */
  int32_t delta;       /* RoPE relocation of the page's keys: logical - stored position */
  int32_t n_valid;     /* keys in the page, P except for the last page of a request */
} rk_entry;

typedef struct {
  int32_t begin, end; /* half-open range of request-local row positions */
} rk_range;

/* Visible state produced by rk_select_visible (all device memory, written
 * by the call).  Table t's entries are entries[entry_start[t] ..
 * entry_start[t] + entry_count[t]), ascending logical_pos: every page of the
 * request that holds at least one key visible to at least one row of the
 * table.  Its rows are the merged ranges ranges[range_start[t] ..
 * + range_count[t]).  The start offsets are fixed by the layout:
 *   entry_start[t] = (layer * Hkv + kvh) * sum_r ceil(L_r / P) + sum_{r'<r} ceil(L_r' / P)
 *   range_start[t] = (layer * Hkv + kvh) * n_segments + (first segment index of r) */
typedef struct {
  rk_entry* entries;    /* [entry_capacity] */
  int32_t* entry_start; /* [n_tables] */
  int32_t* entry_count; /* [n_tables] */
  rk_range* ranges;     /* [range_capacity] */
  int32_t* range_start; /* [n_tables] */
  int32_t* range_count; /* [n_tables] */
  int64_t entry_capacity;
  int64_t range_capacity;
} rk_visible;

typedef struct {
  int64_t n_tables;
  int64_t entry_capacity;  /* rk_entry elements rk_visible.entries must hold */
  int64_t range_capacity;  /* rk_range elements rk_visible.ranges must hold */
  int64_t item_capacity;   /* attention work items the workspace reserves */
  int64_t workspace_bytes; /* device workspace for select + prefill (256-byte aligned) */
} rk_sizes;

/* Validates dims + layout and reports the buffer sizes the other calls need.
 * Host only: touches no GPU.  Errors: RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED. */
rk_status rk_query_sizes(const rk_dims* dims, const rk_layout* layout, rk_sizes* out);

/* SELECTVISIBLESTATE.  Builds, on the GPU, every table's page table and row
 * ranges (bit-exact integer work) plus the attention work list kept in the
 * workspace for rk_segpaged_prefill.  Copies the layout into the workspace
 * (stream-ordered; the host arrays may be reused once the call returns).
 * workspace: device, >= rk_sizes.workspace_bytes, 256-byte aligned; it also
 * holds the device error word, which this call resets.  The layout image is
 * uploaded with cudaMemcpyAsync from a host buffer that the call owns and
 * frees before it returns, so the call is meant to be issued directly on
 * the stream, not recorded into a CUDA graph.
 * Errors (host): RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY,
 * RK_ERR_CUDA.  Device: RK_DEV_BAD_PAGE, RK_DEV_CAPACITY. */
rk_status rk_select_visible(const rk_dims* dims, const rk_layout* layout, const rk_visible* out,
                            void* workspace, size_t workspace_bytes, void* stream);

/* RoPE relocation of cached K pages.  For each job n, with
 * jobs[3n..3n+2] = (src_page, dst_page, delta):
 *   k_dst[dst_page][row][:] = bf16( R(delta) k_src[src_page][row][:] )  for row < P,
 * R the rotate-half RoPE rotation (pairs (m, m + D/2), frequency
 * rope_theta^(-2m/D)), computed in fp32 from angles formed in fp64; delta = 0
 * copies the page bit-exactly.  k_src: device bf16 [n_src_pages][P][D];
 * k_dst: device bf16 [n_dst_pages][P][D] (may be the same pool; a typical use
 * writes R(delta) of each cached page into a working pool at the same page id,
 * leaving the offline store untouched).  jobs: device int32 [n_jobs][3].  A job
 * may read and write the same page; otherwise no page may be written by one
 * job and read or written by another.  Jobs with a page id outside its pool
 * are skipped and set RK_DEV_BAD_PAGE in *device_error (device int32, may be
 * NULL).  Errors (host): RK_ERR_INVALID_ARG, RK_ERR_CUDA. */
rk_status rk_relocate_rope(const void* k_src, int64_t n_src_pages, void* k_dst,
                           int64_t n_dst_pages, const int32_t* jobs, int32_t n_jobs,
                           int32_t page_size, int32_t head_dim, double rope_theta,
                           int32_t* device_error, void* stream);

/* EXECUTE's attention.  For every table's rows i and each q head h of its kv
 * head:  o[layer][tok(i)][h][:] = sum_j softmax_j(softmax_scale <q_i, K'_j>) v_j
 * over the visible keys j of the table, where K'_j is the stored key rotated
 * by its entry's delta when fuse_rope = 1 (fuse_rope = 0: the pool already
 * holds relocated keys and delta is ignored).  bf16 inputs, fp32 accumulation,
 * bf16 output.  Rows outside a table's row set are not written.
 *   q, o: device bf16 [n_layers][T][Hq][D] (token-packed varlen layout)
 *   k_pool, v_pool: device bf16 [n_pages][P][D]; every row of every page
 *     (including rows past n_valid) must hold finite values.
 *   lse: device fp32 [n_layers][Hq][T] natural-log logsumexp, or NULL.
 *   vis, workspace: as filled by rk_select_visible on the same stream.
 * Errors (host): RK_ERR_INVALID_ARG, RK_ERR_CAPACITY, RK_ERR_CUDA.
 * Device: RK_DEV_BAD_PAGE, RK_DEV_TIMEOUT. */
rk_status rk_segpaged_prefill(const rk_dims* dims, const void* q, const void* k_pool,
                              const void* v_pool, const rk_visible* vis, int32_t fuse_rope,
                              double rope_theta, float softmax_scale, void* o, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream);

/* ---- relocation plan (host only) ------------------------------------------
 *
 * The relocate-mode step: rk_relocate_rope rotates, from the K store into a
 * working K pool with the same page ids, every page that a page table lists
 * and that belongs to a cached segment instance with a non-zero delta; then
 * rk_select_visible and rk_segpaged_prefill(fuse_rope = 0) run on a layout
 * whose segments all sit at delta 0 (README excerpt, "Offline KV Reuse +
 * RoPE Relocation"; paooo page, "how to use": BUILDSTATE relocates reused
 * KV, SELECTVISIBLESTATE chooses it).  Attention reads no other page, so no
 * other page needs rotating.  A physical page visible through two instances
 * at different offsets keeps its id for the first instance (in segment
 * order) and gets a fresh run of pages for the later one: the run is
 * appended after the pool (ids n_pages, n_pages + 1, ...) in both the K and
 * the V working pool, filled by K jobs (rotated) and V jobs (delta 0: a
 * copy).  The page tables follow from the layout by the class rule, so the
 * plan is computed on the host from the layout alone. */

typedef struct {
  int64_t n_jobs_k;      /* rk_relocate_rope jobs from the K store into the working K pool */
  int64_t n_jobs_v;      /* jobs within the working V pool (copies into appended pages) */
  int64_t n_extra_pages; /* pages appended to both working pools */
} rk_relocation_sizes;

/* Host only.  Errors: RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY. */
rk_status rk_relocation_query_sizes(const rk_dims* dims, const rk_layout* layout,
                                    rk_relocation_sizes* out);

/* Host only: writes the plan into host buffers.
 *   jobs_k: int32 [cap_k][3] (src_page in the K store, dst_page in the
 *           working K pool, delta); jobs_v: int32 [cap_v][3] (src_page,
 *           dst_page >= n_pages, 0) within the working V pool, whose first
 *           n_pages pages are the caller's V pool.
 *   segments_out [n_segments], page_base_out [n_segments][n_layers * Hkv]:
 *           the relocated layout (every segment at delta 0, appended runs in
 *           page_base); with n_pages + n_extra_pages pages, the same
 *           cu_seqlens, class map, windows and retrieval lists it describes
 *           what the working pools hold.
 * Errors: RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY (cap_k or
 * cap_v below rk_relocation_query_sizes). */
rk_status rk_relocation_plan(const rk_dims* dims, const rk_layout* layout, int32_t* jobs_k,
                             int64_t cap_k, int32_t* jobs_v, int64_t cap_v,
                             rk_segment* segments_out, int32_t* page_base_out);

/* Waits for the stream, then copies the device error word of the workspace
 * into *status (host).  Returns RK_OK when the word is 0, RK_ERR_DEVICE
 * otherwise, RK_ERR_CUDA if the copy failed. */
rk_status rk_get_device_status(const void* workspace, int32_t* status, void* stream);

/* Diagnostic for the kernels' failure detection (the pages have no
 * counterpart): launches one thread that waits, through the same bounded
 * mbarrier wait the attention kernel uses, on a barrier that nothing
 * completes.  After wait_ms milliseconds (1..1000) the wait gives up, ORs
 * RK_DEV_TIMEOUT into *device_word (device int32) and the kernel returns
 * normally; the CUDA context stays usable.  Errors (host): RK_ERR_INVALID_ARG,
 * RK_ERR_CUDA. */
rk_status rk_selftest_bounded_wait(int32_t* device_word, int32_t wait_ms, void* stream);

/* Page tables and row ranges without any device memory from the caller
 * beyond inputs and outputs.  The RedKnot pages have no counterpart of this
 * call; it exists for callers that cannot allocate device memory: code whose
 * framework owns every device allocation through its own pool, or a host
 * thread that must not take the device-wide synchronisation a cudaMalloc can
 * imply.  It computes exactly what rk_select_visible writes into `out`
 * (entries, entry_start/count, ranges, range_start/count); it builds no
 * attention work list, so it cannot feed rk_segpaged_prefill.
 *   - Scratch: a 1 MiB array in the library's device memory (a file-scope
 *     __device__ array, held by every GPU that loads the library until the
 *     process exits) holds the device copy of the layout and the error word.
 *     A layout whose copy does not fit (4 bytes per word of segments,
 *     page_base, cu_seqlens, class map, retrieval lists and per-table work
 *     item offsets, plus about 8.5 KB of fixed fields) is rejected with
 *     RK_ERR_CAPACITY before any GPU work.
 *   - The first call on a device looks up the scratch's device address with
 *     that device current (cudaGetSymbolAddress, once per device); make that
 *     first call before any stream capture on the device.  This note is
 *     about the set-up only and says nothing about whether the call itself
 *     can be captured.
 *   - Every call shares the one scratch array and rewrites all of it that it
 *     reads.  Calls whose GPU work overlaps (other streams, other threads)
 *     race on it: order them on one stream.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * device_error: device int32 (may be NULL) that receives the RK_DEV_* bits of
 * this call.  Errors (host): RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED,
 * RK_ERR_CAPACITY, RK_ERR_CUDA. */
rk_status rk_select_visible_noalloc(const rk_dims* dims, const rk_layout* layout,
                                    const rk_visible* out, int32_t* device_error, void* stream);

/* ---- retrieval page scoring (the retrieval lists of rk_layout) ----------
 *
 * RedKnot's pages say retrieval heads take their cached pages "by query
 * semantics" (paooo page, "how to use" section, SELECTVISIBLESTATE) and give
 * no rule.  These calls implement one reading, for every table (request,
 * layer, kv head) of class RK_RETRIEVAL whose request has uncached rows:
 *   u        = sum over the kv head's q heads of the mean query over the
 *              table's rows (the request's uncached positions);
 *   score_pg = <u, mean over the page's keys of R(delta) K_stored>, for each
 *              candidate page pg: a page of a cached segment whose first
 *              position is at most the last uncached position;
 *   picks    = the top_k candidates by score (ties to the lower page), all
 *              of them when there are at most top_k, in ascending page order.
 * The picks are request-logical page numbers, the format of
 * rk_layout.retr_pages.  Arithmetic: bf16 inputs, fp32 sums, sin / cos of
 * the relocation angle in fp32 after an fp64 reduction modulo 2 pi. */

typedef struct {
  int64_t n_tables;
  int64_t max_pages;       /* pages of the longest request: minimum scores_stride */
  int64_t workspace_bytes; /* device workspace for rk_score_retrieval_pages */
} rk_score_sizes;

/* Validates dims + layout (its retrieval lists may be NULL: scoring makes
 * them) and reports sizes.  top_k: 1 .. 64.  Host only.  Errors:
 * RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY (a table with more
 * than 4096 candidate pages). */
rk_status rk_score_query_sizes(const rk_dims* dims, const rk_layout* layout, int32_t top_k,
                               rk_score_sizes* out);

/* Scores every retrieval table's candidate pages and keeps the top_k.
 *   q:         device bf16 [n_layers][total_tokens][Hq][D], post-RoPE (as for
 *              rk_segpaged_prefill).
 *   k_store:   device bf16 [n_pages][P][D], keys as stored (rotated at their
 *              stored positions; the call relocates by each page's delta).
 *   rope_theta: RoPE base.
 *   out_pages: device int32 [n_tables][top_k]: the picks of table t in
 *              out_pages[t * top_k .. + out_count[t]).
 *   out_count: device int32 [n_tables]: picks per table (0 for other classes
 *              and for tables without rows).
 *   out_scores: device fp32 [n_tables][scores_stride] or NULL: the score of
 *              every candidate page at its page number, NaN elsewhere;
 *              scores_stride >= rk_score_sizes.max_pages.
 *   workspace: device, >= rk_score_sizes.workspace_bytes, 256-byte aligned;
 *              not shared with a concurrent call.
 * Asynchronous on `stream`; the host arrays may be reused once it returns.
 * Errors (host): RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY,
 * RK_ERR_CUDA. */
rk_status rk_score_retrieval_pages(const rk_dims* dims, const rk_layout* layout, const void* q,
                                   const void* k_store, double rope_theta, int32_t top_k,
                                   int32_t* out_pages, int32_t* out_count, float* out_scores,
                                   int64_t scores_stride, void* workspace,
                                   size_t workspace_bytes, void* stream);

/* ---- paged decode -------------------------------------------------------
 *
 * One query row per (request, layer, q head): the last position of each
 * request, a token a decode step appended to the request's uncached tail (its
 * K / V already in the pools).  The row attends to its table's visible keys
 * under the class rule, exactly as the prefill's last row would: global /
 * dense every key, local the last W keys, retrieval the uncached keys and the
 * listed pages.  Reads relocated pools (as rk_segpaged_prefill with
 * fuse_rope = 0) and the page tables rk_select_visible built for the same
 * layout.  bf16 in, fp32 scores and accumulation, bf16 out. */

typedef struct {
  int64_t n_pieces;        /* partial results: the tables' decode pages are cut into equal
                              per-CTA ranges, one partial per (table, range) piece */
  int64_t workspace_bytes; /* device workspace for rk_segpaged_decode */
} rk_decode_sizes;

/* Validates dims + layout and reports the workspace size.  Hq / Hkv <= 8 and
 * n_layers * Hkv <= 1024.  Host only.  Errors: RK_ERR_INVALID_ARG,
 * RK_ERR_UNALIGNED. */
rk_status rk_decode_query_sizes(const rk_dims* dims, const rk_layout* layout,
                                rk_decode_sizes* out);

/*   q:     device bf16 [n_layers][n_req][Hq][D], the new row of each request
 *          (post-RoPE).
 *   k_pool, v_pool: device bf16 [n_pages][P][D], relocated.
 *   vis:   rk_select_visible's output for `layout`.
 *   o:     device bf16 [n_layers][n_req][Hq][D]; entries of a table whose
 *          request's last position is not in its row set (a cached last
 *          segment), or of an empty request, are left untouched.
 *   lse:   device fp32 [n_layers][Hq][n_req] (natural log) or NULL.
 *   workspace: device, >= rk_decode_sizes.workspace_bytes, 256-byte aligned;
 *          its first word is the device error word (RK_DEV_BAD_PAGE), reset
 *          by this call and read by rk_get_device_status.
 * Errors (host): RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY,
 * RK_ERR_CUDA. */
rk_status rk_segpaged_decode(const rk_dims* dims, const rk_layout* layout, const void* q,
                             const void* k_pool, const void* v_pool, const rk_visible* vis,
                             float softmax_scale, void* o, float* lse, void* workspace,
                             size_t workspace_bytes, void* stream);

/* ---- attention importance (sparse FFN token selection) ------------------
 *
 * RedKnot runs the dense FFN only on the tokens with the highest attention
 * scores; the others take the residual path (README "About", Elastic
 * Sparsity / Sparse FFN; paooo page, "main functions").  The pages give no
 * formula.  This call computes, per request r and layer:
 *   I(j) = sum over the layer's q heads h and the rows i that the table of
 *          h's kv head computes of exp(scale q_h(i) . K'_j - lse_h(i)),
 *          0 where j is not visible to i (the class rules of the prefill),
 * i.e. the prefill's attention weights summed over heads and rows, and picks
 * the top_k tokens by I (ties to the lower position), in ascending order.
 * Each computed row's weights sum to one, so the I(j) of a (request, layer)
 * add up to the number of its computed (q head, row) pairs.  fp32
 * accumulation; I is >= 0 (a NaN lse ranks its tokens first). */

typedef struct {
  /* work items: (table, block of 256 page-table keys, row chunk of 4096 / G
   * rows) triples whose rows can see a key of the block; the workspace keeps
   * one 256-float partial sum per item */
  int64_t n_items;
  int64_t workspace_bytes; /* device workspace for rk_attention_importance */
} rk_importance_sizes;

/* Validates dims + layout and reports the workspace size (exact: the items
 * follow from the layout's page tables, which the class rule fixes).
 * Hq / Hkv <= 8 and n_layers * Hkv <= 1024.  Host only.  Errors:
 * RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY (more than 2^23
 * items). */
rk_status rk_importance_query_sizes(const rk_dims* dims, const rk_layout* layout,
                                    rk_importance_sizes* out);

/*   q:      device bf16 [n_layers][T][Hq][D], the prefill's queries.
 *   k_pool: device bf16 [n_pages][P][D], relocated (as rk_segpaged_prefill
 *           with fuse_rope = 0 reads it).
 *   vis:    rk_select_visible's output for `layout`.
 *   lse:    device fp32 [n_layers][Hq][T], natural log: rk_segpaged_prefill's
 *           lse for the same q, pools, layout and softmax_scale.
 *   top_k:  >= 0; tokens picked per (request, layer), min(top_k, L_r).
 *   importance: device fp32 [n_layers][T], written for every position.
 *   tokens: device int32 [n_layers][n_req][top_k], request-local positions,
 *           ascending, the first token_count entries of each row written;
 *           token_count: device int32 [n_layers][n_req].  Both NULL skips
 *           the selection.
 *   workspace: device, >= rk_importance_sizes.workspace_bytes, 256-byte
 *           aligned; its first word is the device error word
 *           (RK_DEV_BAD_PAGE; RK_DEV_CAPACITY if the page tables in `vis`
 *           do not belong to `layout`; RK_DEV_TIMEOUT), reset by this call
 *           and read by rk_get_device_status.  Not shared with a concurrent
 *           call.
 * Errors (host): RK_ERR_INVALID_ARG, RK_ERR_UNALIGNED, RK_ERR_CAPACITY,
 * RK_ERR_CUDA. */
rk_status rk_attention_importance(const rk_dims* dims, const rk_layout* layout, const void* q,
                                  const void* k_pool, const rk_visible* vis, const float* lse,
                                  float softmax_scale, int32_t top_k, float* importance,
                                  int32_t* tokens, int32_t* token_count, void* workspace,
                                  size_t workspace_bytes, void* stream);


/* ---- token-selective FFN (sparse FFN) ------------------------------------
 *
 * RedKnot runs the dense FFN only on the tokens with the highest attention
 * scores and sends the others along the residual path (README "About",
 * Elastic Sparsity / Sparse FFN; paooo page, "main functions").  The pages
 * name the Mistral-7B and Qwen3 families, whose FFN is the gated SiLU MLP;
 * the reading implemented, for each selected row i of the hidden state x:
 *   h   = silu(W_gate x_i) * (W_up x_i)      (d_ff values, rounded to bf16)
 *   x_i = x_i + W_down h                     (fp32 sum, rounded to bf16)
 * and every other row of x is left as it is.  The selection is
 * rk_attention_importance's output for one layer: request r contributes its
 * first min(top_k, L_r) tokens.  bf16 inputs, fp32 accumulation on the
 * tensor cores. */

typedef struct {
  int32_t n_rows;   /* rows of x: the batch's total tokens */
  int32_t d_model;  /* hidden width: a multiple of 256 */
  int32_t d_ff;     /* FFN width: a multiple of 128 */
  int32_t reserved; /* must be 0 */
} rk_ffn_dims;

typedef struct {
  int64_t n_selected;      /* rows the call updates: sum_r min(top_k, L_r) */
  int64_t workspace_bytes; /* device workspace for rk_sparse_ffn */
} rk_ffn_sizes;

/* Validates the shapes and reports the workspace size.  cu_seqlens: host
 * [n_req + 1] (cu_seqlens[0] = 0, non-decreasing, cu_seqlens[n_req] =
 * n_rows).  Host only.  Errors: RK_ERR_INVALID_ARG. */
rk_status rk_ffn_query_sizes(const rk_ffn_dims* dims, int32_t n_req, const int32_t* cu_seqlens,
                             int32_t top_k, rk_ffn_sizes* out);

/*   x:       device bf16 [n_rows][d_model], updated in place at the selected
 *            rows.
 *   tokens:  device int32 [n_req][top_k], request-local positions (the
 *            `tokens` of rk_attention_importance for one layer); the first
 *            min(top_k, L_r) of request r are used and must be distinct.  A
 *            position outside the request is skipped and sets
 *            RK_DEV_BAD_PAGE.
 *   w_gate, w_up: device bf16 [d_ff][d_model]; w_down: device bf16
 *            [d_model][d_ff] (rows are output features, as in a linear
 *            layer's weight).
 *   workspace: device, >= rk_ffn_sizes.workspace_bytes, 256-byte aligned;
 *            its first word is the device error word (RK_DEV_BAD_PAGE,
 *            RK_DEV_TIMEOUT), reset by this call and read by
 *            rk_get_device_status.  It holds the gathered rows and the
 *            bf16 activations h between the two GEMMs.
 * Asynchronous on `stream`.  Errors (host): RK_ERR_INVALID_ARG,
 * RK_ERR_CAPACITY, RK_ERR_CUDA. */
rk_status rk_sparse_ffn(const rk_ffn_dims* dims, int32_t n_req, const int32_t* cu_seqlens,
                        const int32_t* tokens, int32_t top_k, void* x, const void* w_gate,
                        const void* w_up, const void* w_down, void* workspace,
                        size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RK_H_ */
