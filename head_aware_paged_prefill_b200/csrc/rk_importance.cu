// Attention importance for the sparse FFN.  The RedKnot pages run the dense
// FFN only on the tokens with the highest attention scores and send the rest
// along the residual path (README "About", Elastic Sparsity / Sparse FFN;
// paooo page, "main functions" and "core advantages").  They give no
// formula; the reading implemented here, per request and layer:
//   I(j) = sum over the layer's q heads h and the rows i that the table of
//          h's kv head computes of P_h(i, j) = exp(scale q_h(i) . K'_j -
//          lse_h(i)), zero where j is not visible to i,
// that is, the weights the prefill's attention gives each token, summed.  The
// log-sum-exp of every row comes from rk_segpaged_prefill, so one pass over
// the visible pairs suffices.  Then the top k tokens by I, ties to the lower
// position, in ascending order.
//
// Work unit ("item"): one table's block of 256 keys (consecutive entries of
// its page table) against the rows of one row chunk (kImpChunkCols / G
// rows, aligned on row 0) that can see them.  Four launches:
//   1. plan, one CTA per table: the items of the table from its page table
//      and row ranges, written chunk by chunk into the work list at the
//      table's offset (computed on the host from the same rule, and checked
//      here), plus the index arrays the reduction uses.
//   2. column sums, persistent, one CTA per SM, warp-specialised:
//        warp 0    takes items from the list (an atomic counter), loads the
//                  item's 256 keys by TMA (one box per page and 64-column
//                  block) and streams its Q tiles (R = 128 / G rows x the G
//                  q heads of the kv head, one 3-D TMA box per 64 columns)
//                  with their lse, pre-scaled into the log2 domain;
//        warp 1    issues S = K Q^T on the tensor cores (two M = 128 MMAs per
//                  tile, one per half of the keys, N = 128, K = D) into one
//                  of two TMEM buffers;
//        warps 2-9 two warpgroups, one per half of the keys: the thread that
//                  owns a key's TMEM lane adds 2^(S scale log2 e - lse log2 e)
//                  over the tile's columns, masking per element only where a
//                  tile straddles a causal or window edge.  At the item's end
//                  each thread stores its key's sum in the item's slot.
//   3. reduce: every position's importance, adding the slots of its key over
//      kv heads and row chunks in a fixed order (deterministic, no atomics).
//   4. per (request, layer), one 1024-thread CTA: a four-pass radix select
//      on the float bits (all values are >= +0, so the bits order like the
//      values) finds the k-th value; ordered block scans then emit the
//      positions above it and the lowest positions equal to it, ascending.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>

#include "rk_internal.h"
#include "sm100.cuh"

namespace rk {

namespace {

constexpr int kImpSelectThreads = 1024;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kPlanThreads = 256;

constexpr int kKB = kImpKeysPerBlock;  // keys per item (two halves of 128)
constexpr int kColThreads = 320;       // producer, MMA issuer, 8 exponential warps
constexpr int kQStages = 4;
constexpr int kTmemCols = 512;         // two S buffers x two key halves x 128 columns
constexpr uint32_t kNoKey = 0x7fffffffu;

struct ImpArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k_pool;
  const rk_entry* entries;
  const int32_t* entry_start;
  const int32_t* entry_count;
  const rk_range* ranges;
  const int32_t* range_start;
  const int32_t* range_count;
  const int32_t* cu;
  const int2* tplan;    // [n_tables] (list offset, items) from the host
  int2* kbinfo;         // [n_tables][max_kb] (first chunk, last chunk) of a key block
  int2* chunkinfo;      // [n_tables][max_chunks] (list offset in the table, first key block)
  int32_t* inv;         // [n_tables][max_pages] entry index of a request page, -1 if none
  int4* items;          // [n_items] (table, key block, chunk, 0)
  float* part;          // [n_items][kKB]
  const float* lse;
  float* importance;
  int32_t* tokens;
  int32_t* token_count;
  int* work_next;
  int* timeout_site;
  int64_t n_pages;
  int n_req, n_layers, hq, hkv, p, total_tokens, window, top_k;
  int n_items, max_kb, max_chunks, max_pages;
  float scale_log2;
  int8_t cls[kImpMaxLh];
  int32_t* error_word;
};

// ---------------------------------------------------------------------------
// 1. plan
// ---------------------------------------------------------------------------

// First row >= lo and last row <= hi of a table's sorted row ranges (-1 if none).
__device__ __forceinline__ int first_row_at_least(const rk_range* rg, int rc, int lo) {
  for (int x = 0; x < rc; ++x)
    if (rg[x].end > lo) return max(rg[x].begin, lo);
  return -1;
}
__device__ __forceinline__ int last_row_at_most(const rk_range* rg, int rc, int hi) {
  for (int x = rc - 1; x >= 0; --x)
    if (rg[x].begin <= hi) return min(rg[x].end - 1, hi);
  return -1;
}

template <int G>
__global__ void __launch_bounds__(kPlanThreads) importance_plan_kernel(const __grid_constant__ ImpArgs a) {
  constexpr int RPC = kImpChunkCols / G;
  __shared__ int s_off;
  const int t = blockIdx.x, tid = threadIdx.x;
  const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
  const int P = a.p, EPK = kKB / P;
  const int L = a.cu[r + 1] - a.cu[r];
  const int n_e = a.entry_count[t], es = a.entry_start[t];
  const int rc = a.range_count[t];
  const rk_range* rg = a.ranges + a.range_start[t];
  const bool local = a.cls[layer * a.hkv + kvh] == RK_LOCAL;
  const int W = a.window;
  const int npg = (L + P - 1) / P;
  int32_t* inv = a.inv + static_cast<int64_t>(t) * a.max_pages;
  int2* kbi = a.kbinfo + static_cast<int64_t>(t) * a.max_kb;
  int2* chi = a.chunkinfo + static_cast<int64_t>(t) * a.max_chunks;
  const int n_kb = rc > 0 ? (n_e + EPK - 1) / EPK : 0;
  const int n_ch = (L + RPC - 1) / RPC;
  const int2 tp = a.tplan[t];
  for (int pg = tid; pg < npg; pg += kPlanThreads) inv[pg] = -1;
  if (n_kb > a.max_kb || n_ch > a.max_chunks) {  // page tables of another layout
    if (tid == 0) atomicOr(a.error_word, static_cast<int>(RK_DEV_CAPACITY));
    for (int x = tid; x < tp.y; x += kPlanThreads) a.items[tp.x + x] = make_int4(t, -1, 0, 0);
    return;
  }
  __syncthreads();
  for (int e = tid; e < n_e; e += kPlanThreads) {
    const int pg = a.entries[es + e].logical_pos / P;
    if (pg >= 0 && pg < npg) inv[pg] = e;
  }
  for (int kb = tid; kb < n_kb; kb += kPlanThreads) {
    const int e0 = kb * EPK, e1 = min(n_e, e0 + EPK);
    const rk_entry last = a.entries[es + e1 - 1];
    const int pos_lo = a.entries[es + e0].logical_pos;
    const int pos_hi = last.logical_pos + last.n_valid - 1;
    const int hi = local ? min(L - 1, pos_hi + W - 1) : L - 1;
    const int f = first_row_at_least(rg, rc, pos_lo), l = last_row_at_most(rg, rc, hi);
    kbi[kb] = make_int2(f >= 0 ? f / RPC : INT_MAX / 2, l >= 0 ? l / RPC : -1);
  }
  __syncthreads();
  // per chunk c, the key blocks whose chunk range holds c: both ends of the
  // range never decrease with the key block, so they form one run
  for (int c = tid; c < n_ch; c += kPlanThreads) {
    int lo = 0, hi = n_kb;  // first kb with last chunk >= c
    while (lo < hi) {
      const int m = (lo + hi) >> 1;
      if (kbi[m].y >= c) hi = m; else lo = m + 1;
    }
    const int kb_a = lo;
    lo = 0;
    hi = n_kb;  // first kb with first chunk > c
    while (lo < hi) {
      const int m = (lo + hi) >> 1;
      if (kbi[m].x > c) hi = m; else lo = m + 1;
    }
    chi[c] = make_int2(max(0, lo - kb_a), kb_a);  // (count, first kb) for now
  }
  __syncthreads();
  if (tid == 0) {  // exclusive prefix of the per-chunk counts
    int acc = 0;
    for (int c = 0; c < n_ch; ++c) {
      const int2 v = chi[c];
      chi[c] = make_int2(acc, v.y);
      acc += v.x;
    }
    s_off = acc;
  }
  __syncthreads();
  const int total = s_off;
  if (total != tp.y) {  // host and device disagree on the items: write none
    if (tid == 0) atomicOr(a.error_word, static_cast<int>(RK_DEV_CAPACITY));
    for (int x = tid; x < tp.y; x += kPlanThreads) a.items[tp.x + x] = make_int4(t, -1, 0, 0);
    return;
  }
  for (int c = 0; c < n_ch; ++c) {
    const int off = chi[c].x, kb_a = chi[c].y;
    const int cnt = (c + 1 < n_ch ? chi[c + 1].x : total) - off;
    for (int x = tid; x < cnt; x += kPlanThreads)
      a.items[tp.x + off + x] = make_int4(t, kb_a + x, c, 0);
  }
}

// ---------------------------------------------------------------------------
// 2. column sums
// ---------------------------------------------------------------------------

// An item as the producer hands it to the other roles (shared memory).
struct ItemSlot {
  int n_tiles;  // -1: the list is exhausted
  int slot;     // item index = its slot in the partials
  int local;    // 1: local-class window applies
  int pad;
  int kpos[kKB];  // request-local position of each key, kNoKey for none
};

// A Q tile's description and its lse in the log2 domain (shared memory).
struct TileMeta {
  int row0, nrows, pad0, pad1;
  float nl2[128];  // -lse * log2 e of column n = row * G + head, 0 where unused
};

template <int D>
struct ColCfg {
  static constexpr int NCB = D / 64;                  // 64-column blocks
  static constexpr int kHalfBytes = 128 * 128 * NCB;  // 128 keys (or Q rows) x D bf16
  static constexpr int kKBytes = 2 * kHalfBytes;
  static constexpr int kQBytes = kHalfBytes;
  static constexpr int kOffQ = kKBytes;
  static constexpr int kOffMeta = kOffQ + kQStages * kQBytes;
  static constexpr int kOffItem = kOffMeta + kQStages * static_cast<int>(sizeof(TileMeta));
  static constexpr int kOffBar = kOffItem + 2 * static_cast<int>(sizeof(ItemSlot));
  static constexpr int kBytes = kOffBar + 256;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
};

// barrier slots
enum : int {
  kBItemFull = 0,                 // [2] producer lanes (32)
  kBItemEmpty = 2,                // [2] MMA lane + 256 exponential threads
  kBKFull = 4,                    // TMA bytes of the key block
  kBKEmpty = 5,                   // MMAs of the item done (tcgen05.commit)
  kBQFull = 6,                    // [kQStages] producer lanes (32) + Q bytes
  kBQEmpty = 6 + kQStages,        // [kQStages] MMA commit + 256 exponential threads
  kBSFull = 6 + 2 * kQStages,     // [2] tcgen05.commit
  kBSEmpty = 8 + 2 * kQStages,    // [2] 256 exponential threads
  kBDrain = 10 + 2 * kQStages,
  kBCount = 11 + 2 * kQStages,
};

template <int D, int G>
__global__ void __launch_bounds__(kColThreads, 1)
    importance_colsum_kernel(const __grid_constant__ CUtensorMap tm_q,
                             const __grid_constant__ CUtensorMap tm_k,
                             const __grid_constant__ ImpArgs a) {
  using C = ColCfg<D>;
  constexpr int R = 128 / G;      // rows of a Q tile
  constexpr int NV = R * G;       // valid columns of a Q tile (128 when G divides 128)
  constexpr int RPC = kImpChunkCols / G;
  extern __shared__ uint8_t col_raw[];
  uint8_t* sm = col_raw + ((1024 - (smem_u32(col_raw) & 1023)) & 1023);
  uint8_t* sK = sm;
  uint8_t* sQ = sm + C::kOffQ;
  TileMeta* meta = reinterpret_cast<TileMeta*>(sm + C::kOffMeta);
  ItemSlot* islot = reinterpret_cast<ItemSlot*>(sm + C::kOffItem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kBCount);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars[kBItemFull + s], 32);
      mbar_init(&bars[kBItemEmpty + s], 257);
      mbar_init(&bars[kBSFull + s], 1);
      mbar_init(&bars[kBSEmpty + s], 256);
    }
    mbar_init(&bars[kBKFull], 1);
    mbar_init(&bars[kBKEmpty], 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&bars[kBQFull + s], 32);
      mbar_init(&bars[kBQEmpty + s], 257);
    }
    mbar_init(&bars[kBDrain], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, a.error_word, a.timeout_site};
  const int T = a.total_tokens;

  if (warp == 0) {
    // --------------------------------------------------------------- producer
    const int32_t oob_row = static_cast<int32_t>(a.n_pages * a.p);
    const int P = a.p, EPK = kKB / a.p;
    uint32_t q_issued = 0, k_issued = 0;
    uint32_t q_uses[kQStages] = {};
    bool ok = true;
    for (uint32_t it = 0; ok; ++it) {
      const int s = it & 1;
      if (it >= 2 &&
          !(ok = __all_sync(0xffffffffu,
                            mbar_wait(&bars[kBItemEmpty + s], ((it >> 1) - 1) & 1, wc, 1))))
        break;
      int got = 0;
      if (lane == 0) got = atomicAdd(a.work_next, 1);
      got = __shfl_sync(0xffffffffu, got, 0);
      ItemSlot& is = islot[s];
      if (got >= a.n_items) {
        if (lane == 0) is.n_tiles = -1;
        __syncwarp();
        mbar_arrive(&bars[kBItemFull + s]);
        break;
      }
      const int4 w = a.items[got];
      const int t = w.x, kb = w.y, c = w.z;
      const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
      const int t0 = a.cu[r], L = a.cu[r + 1] - t0;
      const int n_e = a.entry_count[t], es = a.entry_start[t];
      const bool local = a.cls[layer * a.hkv + kvh] == RK_LOCAL;
      // the keys: entries kb * EPK .. of the table, P keys each
      const int e0 = kb * EPK, ne = kb >= 0 ? min(EPK, n_e - e0) : 0;
      int pos_lo = INT_MAX, pos_hi = -1;
      for (int k = lane; k < kKB; k += 32) {
        const int e = k / P, row = k % P;
        int kp = static_cast<int>(kNoKey);
        if (e < ne) {
          const rk_entry en = a.entries[es + e0 + e];
          if (en.phys_page >= 0 && en.phys_page < a.n_pages && row < en.n_valid) {
            kp = en.logical_pos + row;
            pos_lo = min(pos_lo, kp);
            pos_hi = max(pos_hi, kp);
          }
        }
        is.kpos[k] = kp;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        pos_lo = min(pos_lo, __shfl_xor_sync(0xffffffffu, pos_lo, o));
        pos_hi = max(pos_hi, __shfl_xor_sync(0xffffffffu, pos_hi, o));
      }
      // the rows of chunk c that can see a key of the block
      const int row_lo = max(pos_lo, c * RPC);
      const int row_hi = min(min(L - 1, local ? pos_hi + a.window - 1 : L - 1), c * RPC + RPC - 1);
      const rk_range* rg = a.ranges + a.range_start[t];
      const int rc = a.range_count[t];
      int n_tiles = 0;
      if (pos_hi >= 0 && row_lo <= row_hi)
        for (int x = 0; x < rc; ++x) {
          const int b0 = max(rg[x].begin, row_lo), b1 = min(rg[x].end, row_hi + 1);
          if (b0 < b1) n_tiles += (b1 - b0 + R - 1) / R;
        }
      if (lane == 0) {
        is.n_tiles = n_tiles;
        is.slot = got;
        is.local = local ? 1 : 0;
      }
      __syncwarp();
      mbar_arrive(&bars[kBItemFull + s]);
      if (n_tiles == 0) continue;
      // the key block: one TMA box per page and 64-column block; missing or
      // bad pages read rows past the pool (zero fill), their keys are masked
      if (k_issued > 0 &&
          !(ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBKEmpty], (k_issued - 1) & 1, wc, 2))))
        break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bars[kBKFull], C::kKBytes);
        for (int e = 0; e < EPK; ++e) {
          int32_t row = oob_row;
          if (e < ne) {
            const int32_t pg = a.entries[es + e0 + e].phys_page;
            if (pg >= 0 && pg < a.n_pages) row = pg * P;
            else atomicOr(a.error_word, static_cast<int>(RK_DEV_BAD_PAGE));
          }
          const int key0 = e * P, half = key0 / 128, rr = key0 % 128;
#pragma unroll
          for (int cb = 0; cb < C::NCB; ++cb)
            tma_load_2d(sK + (half * C::NCB + cb) * (128 * 128) + rr * 128, &tm_k, &bars[kBKFull],
                        cb * 64, row);
        }
      }
      ++k_issued;
      // the Q tiles, range by range
      const float* lse_base = a.lse + (static_cast<int64_t>(layer) * a.hq + kvh * G) * T + t0;
      const int zrow0 = layer * T + t0;
      for (int x = 0; x < rc && ok; ++x) {
        const int b0 = max(rg[x].begin, row_lo), b1 = min(rg[x].end, row_hi + 1);
        for (int row0 = b0; row0 < b1 && ok; row0 += R) {
          const int st = q_issued % kQStages;
          if (q_uses[st] > 0 &&
              !(ok = __all_sync(0xffffffffu,
                                mbar_wait(&bars[kBQEmpty + st], (q_uses[st] - 1) & 1, wc, 3))))
            break;
          const int nrows = min(R, b1 - row0);
          TileMeta& m = meta[st];
          float v[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int n = lane * 4 + u, rr = n / G, h = n - rr * G;
            v[u] = (n < NV && rr < nrows) ? -kLog2e * lse_base[static_cast<int64_t>(h) * T + row0 + rr]
                                          : 0.f;
          }
          *reinterpret_cast<float4*>(&m.nl2[lane * 4]) = make_float4(v[0], v[1], v[2], v[3]);
          if (lane == 0) {
            m.row0 = row0;
            m.nrows = nrows;
            mbar_arrive_expect_tx(&bars[kBQFull + st], C::NCB * NV * 128);
#pragma unroll
            for (int cb = 0; cb < C::NCB; ++cb)
              tma_load_3d(sQ + st * C::kQBytes + cb * (128 * 128), &tm_q, &bars[kBQFull + st],
                          cb * 64, kvh * G, zrow0 + row0);
          } else {
            mbar_arrive(&bars[kBQFull + st]);
          }
          ++q_uses[st];
          ++q_issued;
        }
      }
    }
    // loads still in flight after an abort land before the CTA leaves
    if (lane == 0) {
      if (k_issued > 0) mbar_wait_drain(&bars[kBKFull], (k_issued - 1) & 1);
      for (int st = 0; st < kQStages; ++st)
        if (q_uses[st] > 0) mbar_wait_drain(&bars[kBQFull + st], (q_uses[st] - 1) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 128, false);
      const uint32_t sK_u = smem_u32(sK), sQ_u = smem_u32(sQ);
      uint32_t q_consumed = 0, k_used = 0, tiles = 0;
      bool ok = true;
      for (uint32_t it = 0; ok; ++it) {
        const int s = it & 1;
        if (!(ok = mbar_wait(&bars[kBItemFull + s], (it >> 1) & 1, wc, 4))) break;
        const int n_tiles = islot[s].n_tiles;
        mbar_arrive(&bars[kBItemEmpty + s]);
        if (n_tiles < 0) break;
        if (n_tiles == 0) continue;
        if (!(ok = mbar_wait(&bars[kBKFull], k_used & 1, wc, 5))) break;
        for (int j = 0; j < n_tiles; ++j, ++tiles, ++q_consumed) {
          const int st = q_consumed % kQStages, buf = tiles & 1;
          if (!(ok = mbar_wait(&bars[kBQFull + st], (q_consumed / kQStages) & 1, wc, 6))) break;
          if (tiles >= 2 &&
              !(ok = mbar_wait(&bars[kBSEmpty + buf], ((tiles >> 1) - 1) & 1, wc, 7)))
            break;
          tc_fence_after();
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t ad =
                  desc_sw128(sK_u + (h * C::NCB + (kk >> 2)) * (128 * 128) + (kk & 3) * 32, 16, 1024);
              const uint64_t bd =
                  desc_sw128(sQ_u + st * C::kQBytes + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
              mma_bf16_ss(tmem + buf * 256 + h * 128, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
          tc_commit(&bars[kBSFull + buf]);
          tc_commit(&bars[kBQEmpty + st]);
        }
        if (!ok) break;
        tc_commit(&bars[kBKEmpty]);
        ++k_used;
      }
      // every MMA this thread issued completes before the TMEM is released
      tc_commit(&bars[kBDrain]);
      mbar_wait_drain(&bars[kBDrain], 0);
    }
  } else {
    // ----------------------------------------------------------- exponentials
    const int h = (warp - 2) >> 2;   // key half
    const int quarter = warp & 3;    // TMEM lane quarter this warp may read
    const int key = h * 128 + quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
    const int W = a.window;
    uint32_t q_consumed = 0, tiles = 0;
    bool ok = true;
    for (uint32_t it = 0; ok; ++it) {
      const int s = it & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBItemFull + s], (it >> 1) & 1, wc, 8));
      if (!ok) break;
      const int n_tiles = islot[s].n_tiles, slot = islot[s].slot;
      const bool local = islot[s].local != 0;
      const int kpos = islot[s].kpos[key];
      mbar_arrive(&bars[kBItemEmpty + s]);
      if (n_tiles < 0) break;
      const bool has_key = kpos != static_cast<int>(kNoKey);
      const bool warp_keys = __any_sync(0xffffffffu, has_key);
      uint64_t acc2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
      float accm = 0.f;
      for (int j = 0; j < n_tiles; ++j, ++tiles, ++q_consumed) {
        const int st = q_consumed % kQStages, buf = tiles & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[kBSFull + buf], (tiles >> 1) & 1, wc, 9));
        if (ok)  // the tile's lse landed before the producer's arrivals
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&bars[kBQFull + st], (q_consumed / kQStages) & 1, wc, 10));
        if (!ok) break;
        tc_fence_after();
        const TileMeta& m = meta[st];
        const int row0 = m.row0, nrows = m.nrows;
        const uint32_t taddr = tmem + lane_base + buf * 256 + h * 128;
        const bool open =
            NV == 128 && nrows == R &&
            __all_sync(0xffffffffu, has_key && kpos <= row0 && (!local || row0 + R - 1 - kpos < W));
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t v0[32], v1[32];
          tmem_ld_x32(taddr + half * 64, v0);
          tmem_ld_x32(taddr + half * 64 + 32, v1);
          tmem_ld_wait(v0);
          tmem_ld_wait(v1);
          if (half == 1) {
            tc_fence_before();
            mbar_arrive(&bars[kBSEmpty + buf]);
          }
          if (!warp_keys) continue;
          if (open) {
#pragma unroll
            for (int n = 0; n < 64; n += 4) {
              const float4 l4 = *reinterpret_cast<const float4*>(&m.nl2[half * 64 + n]);
              const uint32_t* v = n < 32 ? v0 : v1;
              const int o = n & 31;
              const uint64_t x0 =
                  f2_fma(f2_pack(__uint_as_float(v[o]), __uint_as_float(v[o + 1])), sc2, f2_pack(l4.x, l4.y));
              const uint64_t x1 = f2_fma(f2_pack(__uint_as_float(v[o + 2]), __uint_as_float(v[o + 3])), sc2,
                                         f2_pack(l4.z, l4.w));
              float p0, p1, p2, p3;
              f2_unpack(x0, p0, p1);
              f2_unpack(x1, p2, p3);
              acc2[0] = f2_add(acc2[0], f2_pack(ex2_approx(p0), ex2_approx(p1)));
              acc2[1] = f2_add(acc2[1], f2_pack(ex2_approx(p2), ex2_approx(p3)));
            }
          } else {
#pragma unroll
            for (int n = 0; n < 64; ++n) {
              const int col = half * 64 + n, rr = col / G, i = row0 + rr;
              const uint32_t* v = n < 32 ? v0 : v1;
              const bool vis = has_key && col < NV && rr < nrows && kpos <= i && (!local || i - kpos < W);
              const float x = fmaf(__uint_as_float(v[n & 31]), a.scale_log2, m.nl2[col]);
              accm += vis ? ex2_approx(x) : 0.f;
            }
          }
        }
        mbar_arrive(&bars[kBQEmpty + st]);
      }
      if (!ok) break;
      float s0, s1, s2, s3;
      f2_unpack(acc2[0], s0, s1);
      f2_unpack(acc2[1], s2, s3);
      a.part[static_cast<int64_t>(slot) * kKB + key] = has_key ? ((s0 + s1) + (s2 + s3)) + accm : 0.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// 3. reduce: I(position) = sum over kv heads, then row chunks, of the slot
// that holds the position's key (fixed order: the result is deterministic)
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(256) importance_reduce_kernel(const __grid_constant__ ImpArgs a) {
  const int pos = blockIdx.x * blockDim.x + threadIdx.x, layer = blockIdx.y;
  if (pos >= a.total_tokens) return;
  int lo = 0, hi = a.n_req;  // request of the position: last r with cu[r] <= pos
  while (hi - lo > 1) {
    const int m = (lo + hi) >> 1;
    if (a.cu[m] <= pos) lo = m; else hi = m;
  }
  const int r = lo, j = pos - a.cu[r], P = a.p;
  float v = 0.f;
  for (int kvh = 0; kvh < a.hkv; ++kvh) {
    const int t = (r * a.n_layers + layer) * a.hkv + kvh;
    const int e = a.inv[static_cast<int64_t>(t) * a.max_pages + j / P];
    if (e < 0) continue;
    const int k = e * P + j % P, kb = k / kKB, kl = k % kKB;
    const int2 cr = a.kbinfo[static_cast<int64_t>(t) * a.max_kb + kb];
    const int list0 = a.tplan[t].x;
    for (int c = cr.x; c <= cr.y; ++c) {
      const int2 ci = a.chunkinfo[static_cast<int64_t>(t) * a.max_chunks + c];
      const int64_t slot = static_cast<int64_t>(list0) + ci.x + kb - ci.y;
      if (slot >= 0 && slot < a.n_items) v += a.part[slot * kKB + kl];
    }
  }
  a.importance[static_cast<int64_t>(layer) * a.total_tokens + pos] = v;
}

// ---------------------------------------------------------------------------
// 4. the top-k tokens of one (request, layer)
// ---------------------------------------------------------------------------

// Exclusive prefix sum over the block (blockDim.x a multiple of 32, <= 1024);
// every thread gets its own exclusive sum and the block total.
__device__ __forceinline__ void block_exclusive_scan(int v, int& excl, int& total, int* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tot[w] = x;
  __syncthreads();
  if (w == 0) {
    int tt = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, tt, o);
      if (lane >= o) tt += y;
    }
    warp_tot[lane] = tt;
  }
  __syncthreads();
  excl = x - v + (w > 0 ? warp_tot[w - 1] : 0);
  total = warp_tot[nw - 1];
  __syncthreads();  // warp_tot is reused by the next scan
}

__global__ void __launch_bounds__(kImpSelectThreads)
    importance_select_kernel(const __grid_constant__ ImpArgs a) {
  __shared__ uint32_t hist[256];
  __shared__ int s_pick[2];
  __shared__ int warp_tot[32];
  const int r = blockIdx.x % a.n_req, layer = blockIdx.x / a.n_req;
  const int t0 = a.cu[r], L = a.cu[r + 1] - t0;
  const float* imp = a.importance + static_cast<int64_t>(layer) * a.total_tokens + t0;
  const int k = min(a.top_k, L);
  if (threadIdx.x == 0 && a.token_count) a.token_count[layer * a.n_req + r] = k;
  if (k <= 0 || !a.tokens) return;
  int32_t* out = a.tokens + (static_cast<int64_t>(layer) * a.n_req + r) * a.top_k;
  const bool all = k >= L;
  uint32_t prefix = 0, mask = 0;
  int need = k;
  if (!all) {
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int x = threadIdx.x; x < 256; x += blockDim.x) hist[x] = 0u;
      __syncthreads();
      for (int pos = threadIdx.x; pos < L; pos += blockDim.x) {
        const uint32_t bits = __float_as_uint(imp[pos]);
        if ((bits & mask) == prefix) atomicAdd(&hist[(bits >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int cum = 0, bin = 255;
        for (; bin > 0; --bin) {
          if (cum + static_cast<int>(hist[bin]) >= need) break;
          cum += static_cast<int>(hist[bin]);
        }
        s_pick[0] = bin;
        s_pick[1] = need - cum;
      }
      __syncthreads();
      prefix |= static_cast<uint32_t>(s_pick[0]) << shift;
      mask |= 255u << shift;
      need = s_pick[1];
      __syncthreads();  // s_pick is rewritten by the next pass
    }
  }
  // prefix now holds the k-th value's bits; take every value above it and the
  // first `need` positions equal to it, in ascending position order
  int eq_base = 0, out_base = 0;
  for (int c0 = 0; c0 < L; c0 += blockDim.x) {
    const int pos = c0 + threadIdx.x;
    const bool in = pos < L;
    const uint32_t bits = in ? __float_as_uint(imp[pos]) : 0u;
    const int eq = (in && !all && bits == prefix) ? 1 : 0;
    int eq_excl, eq_tot;
    block_exclusive_scan(eq, eq_excl, eq_tot, warp_tot);
    const bool sel = in && (all || bits > prefix || (eq && eq_base + eq_excl < need));
    int s_excl, s_tot;
    block_exclusive_scan(sel ? 1 : 0, s_excl, s_tot, warp_tot);
    if (sel && out_base + s_excl < k) out[out_base + s_excl] = pos;  // never past k
    eq_base += eq_tot;
    out_base += s_tot;
  }
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn imp_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

template <int D, int G>
cudaError_t launch_importance_typed(const ImpArgs& a, int n_tables, cudaStream_t stream) {
  using C = ColCfg<D>;
  constexpr int R = 128 / G;
  EncodeTiledFn enc = imp_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  importance_plan_kernel<G><<<n_tables, kPlanThreads, 0, stream>>>(a);
  if (a.n_items > 0) {
    CUtensorMap tq, tk;
    const cuuint64_t qd[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(a.hq),
                              static_cast<cuuint64_t>(a.n_layers) * a.total_tokens};
    const cuuint64_t qs[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(a.hq) * D * 2};
    const cuuint32_t qb[3] = {64, static_cast<cuuint32_t>(G), static_cast<cuuint32_t>(R)};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16*>(a.q), qd, qs, qb,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    const cuuint64_t kd[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(a.n_pages) * a.p};
    const cuuint64_t ks[1] = {static_cast<cuuint64_t>(D) * 2};
    const cuuint32_t kbx[2] = {64, static_cast<cuuint32_t>(a.p)};
    if (enc(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(a.k_pool), kd, ks,
            kbx, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    auto colsum = importance_colsum_kernel<D, G>;
    cudaError_t e = cudaFuncSetAttribute(colsum, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::kAlloc);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return e;
    const int grid = a.n_items < sms ? a.n_items : sms;
    colsum<<<grid, kColThreads, C::kAlloc, stream>>>(tq, tk, a);
  }
  if (a.total_tokens > 0)
    importance_reduce_kernel<<<dim3((a.total_tokens + 255) / 256, a.n_layers), 256, 0, stream>>>(a);
  importance_select_kernel<<<a.n_req * a.n_layers, kImpSelectThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_importance(const ImportanceLaunchArgs& in, cudaStream_t stream) {
  ImpArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(in.q);
  a.k_pool = static_cast<const __nv_bfloat16*>(in.k_pool);
  a.entries = in.entries;
  a.entry_start = in.entry_start;
  a.entry_count = in.entry_count;
  a.ranges = in.ranges;
  a.range_start = in.range_start;
  a.range_count = in.range_count;
  a.cu = in.cu;
  a.tplan = in.tplan;
  a.kbinfo = in.kbinfo;
  a.chunkinfo = in.chunkinfo;
  a.inv = in.inv;
  a.items = in.items;
  a.part = in.part;
  a.lse = in.lse;
  a.importance = in.importance;
  a.tokens = in.tokens;
  a.token_count = in.token_count;
  a.work_next = in.work_next;
  a.timeout_site = in.timeout_site;
  a.n_pages = in.n_pages;
  a.n_req = in.n_req;
  a.n_layers = in.n_layers;
  a.hq = in.hq;
  a.hkv = in.hkv;
  a.p = in.p;
  a.total_tokens = in.total_tokens;
  a.window = in.window;
  a.top_k = in.top_k;
  a.n_items = in.n_items;
  a.max_kb = in.max_kb;
  a.max_chunks = in.max_chunks;
  a.max_pages = in.max_pages;
  a.scale_log2 = in.softmax_scale * kLog2e;
  for (int k = 0; k < in.n_layers * in.hkv; ++k) a.cls[k] = in.cls[k];
  a.error_word = in.error_word;
  const int n_tables = in.n_req * in.n_layers * in.hkv;
  if (n_tables == 0) return cudaSuccess;
  const int G = in.hq / in.hkv;
#define RK_IMP_CASE(DD, GG) \
  if (in.d == DD && G == GG) return launch_importance_typed<DD, GG>(a, n_tables, stream);
  RK_IMP_CASE(128, 1) RK_IMP_CASE(128, 2) RK_IMP_CASE(128, 3) RK_IMP_CASE(128, 4)
  RK_IMP_CASE(128, 5) RK_IMP_CASE(128, 6) RK_IMP_CASE(128, 7) RK_IMP_CASE(128, 8)
  RK_IMP_CASE(64, 1) RK_IMP_CASE(64, 2) RK_IMP_CASE(64, 3) RK_IMP_CASE(64, 4)
  RK_IMP_CASE(64, 5) RK_IMP_CASE(64, 6) RK_IMP_CASE(64, 7) RK_IMP_CASE(64, 8)
#undef RK_IMP_CASE
  return cudaErrorInvalidValue;
}

}  // namespace rk
