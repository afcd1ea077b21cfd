// K1: SELECTVISIBLESTATE on the GPU (RedKnot, paooo page "how to use":
// per request, choose which reused KV each head sees; README excerpt
// "SegPagedAttention Runtime": per-head page table over a segmented store).
//
// One launch, one CTA per table (request, layer, kv_head):
//   1. the ordered page table and the merged row ranges, from the class rule;
//   2. the table's attention work items (<= 128 rows x up to two q heads of
//      one kv head) with the entry range each needs, found by binary search
//      over the table's page positions kept in shared memory; the host gives
//      every table's first item (the item counts follow from the layout);
//   3. the table's item costs (KV tiles) go into a global histogram; the
//      last CTA to finish (a counter in the uploaded layout block) turns it
//      into the first sorted slot of each cost bucket, longest first, and
//      publishes the item count and the selection's error bits in the
//      workspace header.
// Up to kLastCtaSortItems items, the last CTA also moves every item to its
// sorted slot; beyond that a second launch, again one CTA per table, moves
// each table's items (a counting sort spread over all tables: one CTA alone
// took ~0.4 ms for 250K items).
#include <cuda_runtime.h>

#include "rk_internal.h"

namespace rk {

__device__ __forceinline__ const int32_t* lv_arr(const LayoutView* lv, int32_t off) {
  return reinterpret_cast<const int32_t*>(lv) + off;
}

// Exclusive scan of one int per thread across a block of NT threads.
template <int NT>
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, d);
    if (lane >= d) x += y;
  }
  if (lane == 31) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NT / 32 ? warp_tot[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += y;
    }
    if (lane < NT / 32) warp_tot[lane] = w;  // inclusive warp prefix
    if (lane == NT / 32 - 1) *total = w;
  }
  __syncthreads();
  int excl = x - v + (warp > 0 ? warp_tot[warp - 1] : 0);
  __syncthreads();
  return excl;
}

constexpr int kSelectThreads = 512;
static_assert(kCostBuckets % kSelectThreads == 0, "buckets per thread");
constexpr int kLastCtaSortItems = 16384;
constexpr int kScatterBatch = 4;  // items a thread loads before claiming their slots
constexpr int kPosCap = 3072;  // page positions of one table kept in shared memory

// Claims one slot of counter hist[b] per lane; lanes of the warp with the
// same b share one atomic (a cost bucket is often shared by hundreds of
// items).  Every lane of the warp must call it; lanes with valid == false
// take no slot.  Returns the old counter value plus this lane's rank.
__device__ __forceinline__ int warp_claim(int* hist, int b, bool valid) {
  const int key = valid ? b : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, key);
  const int lane = threadIdx.x & 31;
  const int leader = __ffs(peers) - 1;
  const int rank = __popc(peers & ((1u << lane) - 1u));
  int base = 0;
  if (valid && lane == leader) base = atomicAdd(&hist[b], __popc(peers));
  base = __shfl_sync(0xffffffffu, base, leader);
  return base + rank;
}

// bucket of an item: groups in order ((request, layer) groups when the
// layout has several), the longest first inside a group
__device__ __forceinline__ int item_bucket(const LayoutView* lv, int req, int layer, int cost) {
  const int groups = lv->bucket_groups;
  const int bpg = kCostBuckets / groups;
  const int g = groups > 1 ? req * lv->n_layers + layer : 0;
  const int c = min(max(cost, 0) / lv->cost_width, bpg - 1);
  return g * bpg + (bpg - 1 - c);
}

// index of the first of n entries whose key exceeds v (keys ascending)
template <typename Key>
__device__ __forceinline__ int upper_bound(int n, int v, Key key) {
  int a = 0, b = n;
  while (a < b) {
    const int mid = (a + b) >> 1;
    if (key(mid) <= v) a = mid + 1; else b = mid;
  }
  return a;
}

__global__ void __launch_bounds__(kSelectThreads)
    select_kernel(LayoutView* __restrict__ lv, rk_visible vis, WsHeader* hdr, Item* items_tmp,
                  int32_t* cursor, Item* items) {
  __shared__ int warp_tot[kSelectThreads / 32];
  __shared__ int s_total;
  __shared__ int s_last;
  __shared__ int hist[kCostBuckets];
  __shared__ int2 s_pos[kPosCap];  // (logical_pos, n_valid) of the table's entries
  const int t = blockIdx.x;
  const int hkv = lv->hkv, n_layers = lv->n_layers, P = lv->p;
  const int kvh = t % hkv, layer = (t / hkv) % n_layers, r = t / (hkv * n_layers);
  const int lh = layer * hkv + kvh;
  const int n_lh = n_layers * hkv;
  const int32_t* seg = lv_arr(lv, lv->off_seg);
  const int32_t* seg_indptr = lv_arr(lv, lv->off_seg_indptr);
  const int32_t* page_base = lv_arr(lv, lv->off_page_base);
  const int32_t* cu = lv_arr(lv, lv->off_cu);
  const int32_t* page_prefix = lv_arr(lv, lv->off_page_prefix);
  const int32_t* cls_arr = lv_arr(lv, lv->off_class);
  const int32_t* retr_indptr = lv_arr(lv, lv->off_retr_indptr);
  const int32_t* retr_pages = lv_arr(lv, lv->off_retr_pages);
  const int32_t* tile_prefix = lv_arr(lv, lv->off_tile_prefix);

  const int L = cu[r + 1] - cu[r];
  const int npg = (L + P - 1) / P;
  const int cls = cls_arr[lh];
  const int W = lv->window;
  const int s0 = seg_indptr[r], s1 = seg_indptr[r + 1];
  const int estart = lh * lv->total_pages + page_prefix[r];
  const int rstart = lh * lv->n_seg + s0;
  const int rb = retr_indptr[t], re = retr_indptr[t + 1];

  // last uncached position of the request (-1 if none)
  int last_unc = -1;
  for (int s = s0; s < s1; ++s)
    if (!seg[5 * s + 4]) last_unc = max(last_unc, seg[5 * s + 1] + seg[5 * s + 2] - 1);

  // ---- 1. page table
  int count = 0;
  for (int base = 0; base < npg; base += kSelectThreads) {
    const int k = base + threadIdx.x;
    int flag = 0;
    rk_entry e{0, 0, 0, 0};
    if (k < npg) {
      const int pos = k * P;
      const int nv = min(P, L - pos);
      // segment holding pos: last s in [s0, s1) with start <= pos
      int lo = s0, hi = s1 - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (seg[5 * mid + 1] <= pos) lo = mid; else hi = mid - 1;
      }
      const int s = lo;
      const int start = seg[5 * s + 1];
      const bool cached = seg[5 * s + 4] != 0;
      if (cls == RK_GLOBAL || cls == RK_DENSE) {
        flag = 1;
      } else if (cls == RK_LOCAL) {
        // rows of an uncached segment [a, b) see keys [a - W + 1, b - 1]
        for (int u = s0; u < s1 && !flag; ++u) {
          if (seg[5 * u + 4]) continue;
          const int a = seg[5 * u + 1], b = a + seg[5 * u + 2];
          flag = max(pos, a - W + 1) <= min(pos + nv - 1, b - 1);
        }
      } else {  // retrieval: uncached pages, and listed cached pages before the last row
        if (!cached) {
          flag = 1;
        } else if (pos <= last_unc) {
          for (int x = rb; x < re && !flag; ++x) flag = retr_pages[x] == k;
        }
      }
      if (flag) {
        const int pis = (pos - start) / P;
        int64_t phys = static_cast<int64_t>(page_base[static_cast<int64_t>(s) * n_lh + lh]) + pis;
        if (phys < 0 || phys >= lv->n_pages) atomicOr(&lv->error, static_cast<int>(RK_DEV_BAD_PAGE));
        e.phys_page = static_cast<int32_t>(phys);
        e.logical_pos = pos;
        e.delta = start - seg[5 * s + 3];
        e.n_valid = nv;
      }
    }
    const int off = block_exclusive_scan<kSelectThreads>(flag, warp_tot, &s_total);
    if (flag) {
      vis.entries[estart + count + off] = e;
      if (count + off < kPosCap) s_pos[count + off] = make_int2(e.logical_pos, e.n_valid);
    }
    count += s_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    vis.entry_start[t] = estart;
    vis.entry_count[t] = count;
    int n = 0;
    if (cls == RK_GLOBAL || cls == RK_DENSE) {
      if (L > 0) {
        vis.ranges[rstart] = rk_range{0, L};
        n = 1;
      }
    } else {
      int cur_b = -1, cur_e = -1;
      for (int s = s0; s < s1; ++s) {
        if (seg[5 * s + 4]) continue;
        const int a = seg[5 * s + 1], b = a + seg[5 * s + 2];
        if (n > 0 && cur_e == a) {
          cur_e = b;
          vis.ranges[rstart + n - 1].end = b;
        } else {
          cur_b = a;
          cur_e = b;
          vis.ranges[rstart + n] = rk_range{cur_b, cur_e};
          ++n;
        }
      }
    }
    vis.range_start[t] = rstart;
    vis.range_count[t] = n;
    s_total = n;
  }
  __syncthreads();

  // ---- 2. this table's work items
  if (items_tmp) {
    const int n_rng = s_total;
    const int G = lv->hq / hkv;
    const int npairs = (G + 1) / 2;
    const int ept = kKeysPerTile / P;
    const int T = lv->total_tokens;
    const int first = tile_prefix[t], n_it = tile_prefix[t + 1] - first;
    const rk_entry* E = vis.entries + estart;
    const bool in_smem = count <= kPosCap;
    auto lp = [&](int m) { return in_smem ? s_pos[m].x : E[m].logical_pos; };
    auto last_key = [&](int m) {
      return in_smem ? s_pos[m].x + s_pos[m].y - 1 : E[m].logical_pos + E[m].n_valid - 1;
    };
    for (int k = threadIdx.x; k < kCostBuckets; k += kSelectThreads) hist[k] = 0;
    __syncthreads();
    // all lanes run every round (warp_claim is warp-collective)
    const int rounds = (n_it + kSelectThreads - 1) / kSelectThreads;
    for (int round = 0; round < rounds; ++round) {
      const int x = round * kSelectThreads + threadIdx.x;
      int bucket = -1;
      if (x < n_it) {
        const int pair = x % npairs;
        int tile = x / npairs;
        int rbeg = 0, rend = 0;
        for (int k = 0; k < n_rng; ++k) {
          const rk_range rg = vis.ranges[rstart + k];
          const int nt = (rg.end - rg.begin + kRowsPerTile - 1) / kRowsPerTile;
          if (tile < nt) {
            rbeg = rg.begin + tile * kRowsPerTile;
            rend = min(rbeg + kRowsPerTile, rg.end);
            break;
          }
          tile -= nt;
        }
        // entries whose first key is at most the tile's last row
        const int e_hi = upper_bound(count, rend - 1, lp);
        int e_lo = 0, window = -1;
        if (cls == RK_LOCAL) {
          // first entry whose last key reaches the first row's window start
          window = W;
          e_lo = upper_bound(e_hi, rbeg - W, last_key);
        }
        Item it;
        it.q_row0 = layer * T + cu[r];
        it.row_begin = rbeg;
        it.row_end = rend;
        it.e_begin = estart + e_lo;
        it.e_end = estart + e_hi;
        it.qh0 = kvh * G + 2 * pair;
        it.nh = min(2, G - 2 * pair);
        it.window = window;
        it.layer = layer;
        it.req = r;
        it.table = t;
        it.cost = (e_hi - e_lo + ept - 1) / ept;
        items_tmp[first + x] = it;
        bucket = item_bucket(lv, r, layer, it.cost);
      }
      warp_claim(hist, bucket, bucket >= 0);
    }
    __syncthreads();
    int* g_hist = const_cast<int*>(lv_arr(lv, lv->off_cost_hist));
    for (int k = threadIdx.x; k < kCostBuckets; k += kSelectThreads)
      if (hist[k]) atomicAdd(&g_hist[k], hist[k]);
  }

  // ---- 3. the last CTA turns the cost histogram into bucket slots and publishes the header
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(&lv->done_count, 1) == static_cast<int>(gridDim.x) - 1;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  const int total = items_tmp ? tile_prefix[gridDim.x] : 0;
  if (items_tmp) {
    // first sorted slot of each bucket, kCostBuckets / kSelectThreads per thread
    const int* g_hist = lv_arr(lv, lv->off_cost_hist);
    constexpr int per = kCostBuckets / kSelectThreads;
    int loc[per];
    int sum = 0;
#pragma unroll
    for (int k = 0; k < per; ++k) {
      loc[k] = __ldcg(&g_hist[threadIdx.x * per + k]);
      sum += loc[k];
    }
    const int ex = block_exclusive_scan<kSelectThreads>(sum, warp_tot, &s_total);
    int run = ex;
    // items given: this CTA sorts them, with the cursors in shared memory
    int* cur = items ? hist : cursor;
#pragma unroll
    for (int k = 0; k < per; ++k) {
      cur[threadIdx.x * per + k] = run;
      run += loc[k];
    }
    if (items) {
      __syncthreads();
      constexpr int kChunk = kSelectThreads * kScatterBatch;
      for (int base = 0; base < total; base += kChunk) {
        Item it[kScatterBatch];
#pragma unroll
        for (int b = 0; b < kScatterBatch; ++b) {
          const int x = base + b * kSelectThreads + threadIdx.x;
          if (x < total) it[b] = items_tmp[x];
        }
#pragma unroll
        for (int b = 0; b < kScatterBatch; ++b) {
          const int x = base + b * kSelectThreads + threadIdx.x;
          const bool v = x < total;
          const int pos =
              warp_claim(hist, v ? item_bucket(lv, it[b].req, it[b].layer, it[b].cost) : 0, v);
          if (v) items[pos] = it[b];
        }
      }
    }
  }
  if (threadIdx.x == 0) {
    hdr->n_items = total;
    hdr->timeout_site = 0;
    hdr->work_next = 0;
    hdr->work_done = 0;
    hdr->error = *reinterpret_cast<volatile int*>(&lv->error);
  }
}

// Second launch: one CTA per table moves the table's items to their slots in
// the cost order (within a bucket the order is arbitrary).
__global__ void __launch_bounds__(kSelectThreads)
    scatter_kernel(const LayoutView* __restrict__ lv, const Item* __restrict__ items_tmp,
                   Item* __restrict__ items, int32_t* cursor) {
  __shared__ int hist[kCostBuckets];
  const int32_t* tile_prefix = lv_arr(lv, lv->off_tile_prefix);
  const int first = tile_prefix[blockIdx.x], n_it = tile_prefix[blockIdx.x + 1] - first;
  if (n_it <= 0) return;
  for (int k = threadIdx.x; k < kCostBuckets; k += kSelectThreads) hist[k] = 0;
  __syncthreads();
  const int rounds = (n_it + kSelectThreads - 1) / kSelectThreads;
  for (int round = 0; round < rounds; ++round) {
    const int x = round * kSelectThreads + threadIdx.x;
    const bool v = x < n_it;
    const Item* ix = items_tmp + first + x;
    warp_claim(hist, v ? item_bucket(lv, ix->req, ix->layer, ix->cost) : 0, v);
  }
  __syncthreads();
  // this table's run of each bucket
  for (int k = threadIdx.x; k < kCostBuckets; k += kSelectThreads)
    if (hist[k]) hist[k] = atomicAdd(&cursor[k], hist[k]);
  __syncthreads();
  for (int round = 0; round < rounds; ++round) {
    const int x = round * kSelectThreads + threadIdx.x;
    const bool v = x < n_it;
    Item it;
    if (v) it = items_tmp[first + x];
    const int pos = warp_claim(hist, v ? item_bucket(lv, it.req, it.layer, it.cost) : 0, v);
    if (v) items[pos] = it;
  }
}

cudaError_t launch_select(LayoutView* lv_dev, int n_tables, const rk_visible& vis, WsHeader* hdr,
                          Item* items_tmp, Item* items, int32_t* cursor, int64_t n_items,
                          cudaStream_t stream) {
  if (n_tables <= 0) return cudaSuccess;
  if (n_items <= kLastCtaSortItems) {
    select_kernel<<<n_tables, kSelectThreads, 0, stream>>>(lv_dev, vis, hdr, items_tmp, cursor,
                                                           items);
  } else {
    select_kernel<<<n_tables, kSelectThreads, 0, stream>>>(lv_dev, vis, hdr, items_tmp, cursor,
                                                           nullptr);
    scatter_kernel<<<n_tables, kSelectThreads, 0, stream>>>(lv_dev, items_tmp, items, cursor);
  }
  return cudaGetLastError();
}

// Page-table stage alone (no work list), for the no-allocation entry point.
cudaError_t launch_select_tables_only(LayoutView* lv_dev, int n_tables, const rk_visible& vis,
                                      WsHeader* hdr, cudaStream_t stream) {
  if (n_tables > 0)
    select_kernel<<<n_tables, kSelectThreads, 0, stream>>>(lv_dev, vis, hdr, nullptr, nullptr,
                                                           nullptr);
  return cudaGetLastError();
}

}  // namespace rk
