// K1: SELECTVISIBLESTATE on the GPU (RedKnot, paooo page "how to use":
// per request, choose which reused KV each head sees; README excerpt
// "SegPagedAttention Runtime": per-head page table over a segmented store).
//
// select_tables_kernel : one CTA per table (request, layer, kv_head) derives
//   the ordered page table and the merged row ranges from the class rules.
// build_worklist_kernel: one CTA turns the tables into attention work items
//   (<= 128 rows x up to two q heads of one kv head) with the entry range each
//   item needs, sorted by cost (KV tiles), longest first.
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

constexpr int kSelectThreads = 256;

__global__ void __launch_bounds__(kSelectThreads)
    select_tables_kernel(const LayoutView* __restrict__ lv, rk_visible vis, WsHeader* hdr) {
  __shared__ int warp_tot[kSelectThreads / 32];
  __shared__ int s_total;
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
        if (phys < 0 || phys >= lv->n_pages) {
          atomicOr(&hdr->error, static_cast<int>(RK_DEV_BAD_PAGE));
        }
        e.phys_page = static_cast<int32_t>(phys);
        e.logical_pos = pos;
        e.delta = start - seg[5 * s + 3];
        e.n_valid = nv;
      }
    }
    const int off = block_exclusive_scan<kSelectThreads>(flag, warp_tot, &s_total);
    if (flag) vis.entries[estart + count + off] = e;
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
  }
}

constexpr int kWorklistThreads = 1024;
constexpr int kCostBuckets = 4096;

__global__ void __launch_bounds__(kWorklistThreads)
    build_worklist_kernel(LayoutView* lv, rk_visible vis, WsHeader* hdr, Item* items_tmp,
                          Item* items) {
  __shared__ int warp_tot[kWorklistThreads / 32];
  __shared__ int s_total;
  __shared__ int hist[kCostBuckets];
  const int hkv = lv->hkv, n_layers = lv->n_layers, P = lv->p;
  const int n_tables = lv->n_req * n_layers * hkv;
  const int G = lv->hq / hkv;
  const int npairs = (G + 1) / 2;
  const int ept = kKeysPerTile / P;
  const int W = lv->window;
  const int T = lv->total_tokens;
  int32_t* tile_prefix = reinterpret_cast<int32_t*>(lv) + lv->off_tile_prefix;
  const int32_t* cu = lv_arr(lv, lv->off_cu);
  const int32_t* cls_arr = lv_arr(lv, lv->off_class);

  // items per table
  for (int t = threadIdx.x; t < n_tables; t += kWorklistThreads) {
    const int rs = vis.range_start[t], rn = vis.range_count[t];
    int tiles = 0;
    for (int x = 0; x < rn; ++x) {
      const rk_range rg = vis.ranges[rs + x];
      tiles += (rg.end - rg.begin + kRowsPerTile - 1) / kRowsPerTile;
    }
    tile_prefix[t + 1] = tiles * npairs;
  }
  __syncthreads();
  // exclusive prefix over tables
  int carry = 0;
  for (int base = 0; base < n_tables; base += kWorklistThreads) {
    const int t = base + threadIdx.x;
    const int v = t < n_tables ? tile_prefix[t + 1] : 0;
    const int ex = block_exclusive_scan<kWorklistThreads>(v, warp_tot, &s_total);
    if (t < n_tables) tile_prefix[t] = carry + ex;
    carry += s_total;
    __syncthreads();
  }
  if (threadIdx.x == 0) tile_prefix[n_tables] = carry;
  __syncthreads();
  const int total = carry;
  if (total > lv->item_capacity) {
    if (threadIdx.x == 0) {
      atomicOr(&hdr->error, static_cast<int>(RK_DEV_CAPACITY));
      hdr->n_items = 0;
    }
    return;
  }

  for (int b = threadIdx.x; b < kCostBuckets; b += kWorklistThreads) hist[b] = 0;
  __syncthreads();

  for (int x = threadIdx.x; x < total; x += kWorklistThreads) {
    // table of item x: last t with tile_prefix[t] <= x
    int lo = 0, hi = n_tables - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tile_prefix[mid] <= x) lo = mid; else hi = mid - 1;
    }
    const int t = lo;
    const int kvh = t % hkv, layer = (t / hkv) % n_layers, r = t / (hkv * n_layers);
    const int local = x - tile_prefix[t];
    const int pair = local % npairs;
    int tile = local / npairs;
    const int rs = vis.range_start[t], rn = vis.range_count[t];
    int rbeg = 0, rend = 0;
    for (int k = 0; k < rn; ++k) {
      const rk_range rg = vis.ranges[rs + k];
      const int nt = (rg.end - rg.begin + kRowsPerTile - 1) / kRowsPerTile;
      if (tile < nt) {
        rbeg = rg.begin + tile * kRowsPerTile;
        rend = min(rbeg + kRowsPerTile, rg.end);
        break;
      }
      tile -= nt;
    }
    const int es = vis.entry_start[t], en = vis.entry_count[t];
    const rk_entry* E = vis.entries + es;
    // e_hi: first entry whose page starts after the tile's last row
    int a = 0, b = en;
    while (a < b) {
      const int mid = (a + b) >> 1;
      if (E[mid].logical_pos <= rend - 1) a = mid + 1; else b = mid;
    }
    const int e_hi = a;
    const int cls = cls_arr[layer * hkv + kvh];
    int e_lo = 0;
    int window = -1;
    if (cls == RK_LOCAL) {
      window = W;
      // first entry whose last key reaches the first row's window start
      const int first_key = rbeg - W + 1;
      a = 0;
      b = e_hi;
      while (a < b) {
        const int mid = (a + b) >> 1;
        if (E[mid].logical_pos + E[mid].n_valid - 1 < first_key) a = mid + 1; else b = mid;
      }
      e_lo = a;
    }
    Item it;
    it.q_row0 = layer * T + cu[r];
    it.row_begin = rbeg;
    it.row_end = rend;
    it.e_begin = es + e_lo;
    it.e_end = es + e_hi;
    it.qh0 = kvh * G + 2 * pair;
    it.nh = min(2, G - 2 * pair);
    it.window = window;
    it.layer = layer;
    it.req = r;
    it.table = t;
    it.cost = (e_hi - e_lo + ept - 1) / ept;
    items_tmp[x] = it;
    atomicAdd(&hist[kCostBuckets - 1 - min(it.cost, kCostBuckets - 1)], 1);
  }
  __syncthreads();
  // bucket offsets (descending cost order), 4 buckets per thread
  {
    constexpr int per = kCostBuckets / kWorklistThreads;
    int loc[per];
    int sum = 0;
#pragma unroll
    for (int k = 0; k < per; ++k) {
      loc[k] = hist[threadIdx.x * per + k];
      sum += loc[k];
    }
    const int ex = block_exclusive_scan<kWorklistThreads>(sum, warp_tot, &s_total);
    int run = ex;
#pragma unroll
    for (int k = 0; k < per; ++k) {
      hist[threadIdx.x * per + k] = run;
      run += loc[k];
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < total; x += kWorklistThreads) {
    const Item it = items_tmp[x];
    const int pos = atomicAdd(&hist[kCostBuckets - 1 - min(it.cost, kCostBuckets - 1)], 1);
    items[pos] = it;
  }
  if (threadIdx.x == 0) hdr->n_items = total;
}

cudaError_t launch_select(LayoutView* lv_dev, int n_tables, const rk_visible& vis, WsHeader* hdr,
                          Item* items_tmp, Item* items, cudaStream_t stream) {
  if (n_tables > 0) {
    select_tables_kernel<<<n_tables, kSelectThreads, 0, stream>>>(lv_dev, vis, hdr);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  build_worklist_kernel<<<1, kWorklistThreads, 0, stream>>>(lv_dev, vis, hdr, items_tmp, items);
  return cudaGetLastError();
}

// Page-table stage alone (no work list), for the no-allocation entry point.
cudaError_t launch_select_tables_only(LayoutView* lv_dev, int n_tables, const rk_visible& vis,
                                      WsHeader* hdr, cudaStream_t stream) {
  if (n_tables > 0) select_tables_kernel<<<n_tables, kSelectThreads, 0, stream>>>(lv_dev, vis, hdr);
  return cudaGetLastError();
}

}  // namespace rk
