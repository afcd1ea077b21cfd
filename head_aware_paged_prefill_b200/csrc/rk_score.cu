// Retrieval page scoring: each retrieval head's cached pages ranked against
// its queries, the top k kept for rk_select_visible's retrieval lists.
//
// RedKnot's pages say retrieval heads take their cached pages "by query
// semantics" (paooo page, "how to use" section, SELECTVISIBLESTATE) and give
// no rule.  The reading implemented, per retrieval table (request, layer,
// kv head) with rows:
//   u        = sum over the kv head's q heads of the mean query over the
//              table's rows (its uncached positions);
//   score_pg = <u, mean over the page's keys of R(delta) K_stored>
//            = <R(-delta) u, mean over the page's keys of K_stored>,
//              so the key means need no rotation and u is rotated once per
//              run of candidates sharing a delta (a cached segment);
//   picks    = the top k candidate pages (cached, starting at or before the
//              last row), ties to the lower page, ascending page order.
//
// The host describes a table's candidates by runs (the pages of one cached
// segment that start at or before the last row) and its query rows by the
// request's uncached ranges; the kernel expands both.  One persistent launch
// (a few CTAs per SM) walks a list of equal-sized work units:
//   - a query unit sums the queries of one 64-row chunk of a table over the
//     kv head's q heads (fp32, fixed order, 16-byte loads);
//   - a page unit averages the stored keys of 4 candidate pages, four warps
//     per page (a quarter of its rows each), combined in a fixed order.
// Every unit bumps its table's counter; the CTA that finishes a table's last
// unit ranks the table at once: u from the chunk sums (in chunk order),
// R(-delta) u per run, one warp per candidate for its dot product, then each
// candidate's rank as the number of (score, page) keys above its own (a
// bitonic sort above 2048 candidates); the first k, in ascending page order,
// are the picks.  Streaming (HBM bound) and ranking of different tables
// overlap, and the ranking reads data the same launch just wrote to L2.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "rk_internal.h"

namespace rk {

namespace {

__device__ __forceinline__ const int32_t* sv_arr(const ScoreView* sv, int32_t off) {
  return reinterpret_cast<const int32_t*>(sv) + off;
}

struct ScoreFreqs {
  double f[64];  // theta^(-2m/D), m < D/2
};

constexpr int kScoreThreads = 512;
constexpr int kScoreWarps = kScoreThreads / 32;
constexpr int kWarpsPerPage = kScoreWarps / kScorePagesPerUnit;
static_assert(kWarpsPerPage * kScorePagesPerUnit == kScoreWarps, "warps per page");
constexpr int kRankCount = 2048;  // candidates ranked by counting (a sort above)
constexpr int kRankBatch = 16;    // candidates a warp loads before reducing

template <int D>
struct ScoreSmem {
  // unit phase
  static constexpr int kAccBytes = (kScoreThreads / (D / 8)) * D * 4;  // query slots x D
  static constexpr int kRedBytes = kScoreWarps * D * 4;               // page partials
  static constexpr int kUnitBytes = kAccBytes > kRedBytes ? kAccBytes : kRedBytes;
  // rank phase
  static constexpr int kOffKey = 0;                                  // u64 [kScoreMaxCand]
  static constexpr int kOffPicked = kOffKey + 8 * kScoreMaxCand;     // int [kRankCount]
  static constexpr int kOffU = kOffPicked + 4 * kRankCount;          // float [D]
  static constexpr int kOffRed = kOffU + 4 * D;                      // float [threads / D][D]
  static constexpr int kRankBytes = kOffRed + 4 * kScoreThreads;
  static constexpr int kBytes = kUnitBytes > kRankBytes ? kUnitBytes : kRankBytes;
};

__device__ __forceinline__ uint32_t order_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// Last index in [lo, hi) whose key is <= x (the keys ascend; lo's is <= x).
template <typename F>
__device__ __forceinline__ int last_at_most(int lo, int hi, int x, F key) {
  while (hi - lo > 1) {
    const int m = (lo + hi) >> 1;
    if (key(m) <= x) lo = m; else hi = m;
  }
  return lo;
}

// Query unit: thread (slot, column group) adds 8 consecutive columns (one
// 16-byte load) of the (row, head) pairs slot, slot + S, ...; the slots are
// then added in order.
template <int D>
__device__ void query_unit(const ScoreView* sv, const ScoreTable& st, int chunk,
                           const __nv_bfloat16* __restrict__ q, float* __restrict__ partials,
                           uint8_t* smem) {
  constexpr int CG = D / 8, S = kScoreThreads / CG;
  float(*acc_s)[D] = reinterpret_cast<float(*)[D]>(smem);
  const ScoreRange* rgs = reinterpret_cast<const ScoreRange*>(sv_arr(sv, sv->off_ranges));
  int lc = chunk - st.chunk_begin, row_begin = 0, n_rows = 0;
  for (int x = st.range_begin; x < st.range_end; ++x) {
    const int len = rgs[x].end - rgs[x].begin;
    const int nck = (len + kScoreChunkRows - 1) / kScoreChunkRows;
    if (lc < nck) {
      row_begin = rgs[x].begin + lc * kScoreChunkRows;
      n_rows = min(kScoreChunkRows, rgs[x].end - row_begin);
      break;
    }
    lc -= nck;
  }
  const int g = sv->g, hq = sv->hq;
  const int cg = threadIdx.x % CG, slot = threadIdx.x / CG;
  const int n_pairs = n_rows * g;
  float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
  for (int pr = slot; pr < n_pairs; pr += S) {
    const int i = pr / g, h = pr - i * g;
    const int64_t row = static_cast<int64_t>(st.q_row0) + row_begin + i;
    const uint4 raw = *reinterpret_cast<const uint4*>(q + (row * hq + st.head0 + h) * D + cg * 8);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 v = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[k]));
      a[2 * k] += v.x;
      a[2 * k + 1] += v.y;
    }
  }
#pragma unroll
  for (int k = 0; k < 8; ++k) acc_s[slot][cg * 8 + k] = a[k];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kScoreThreads) {
    float t = 0.f;
    for (int sl = 0; sl < S; ++sl) t += acc_s[sl][c];
    partials[static_cast<int64_t>(chunk) * D + c] = t;
  }
}

// Page unit: candidates [c0, c0 + 4) of a table; warp w takes candidate
// w / kWarpsPerPage and the rows of its quarter, each lane D / 32 columns of
// every key row; the quarters are added in order.
template <int D>
__device__ void page_unit(const ScoreTable& st, const ScoreRun* runs, int c0,
                          const __nv_bfloat16* __restrict__ k_store, int P,
                          float* __restrict__ kbar, uint8_t* smem) {
  constexpr int CPL = D / 32;
  float(*red)[D] = reinterpret_cast<float(*)[D]>(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cl = warp / kWarpsPerPage, qr = warp % kWarpsPerPage;
  const int c = c0 + cl;
  auto run_key = [&](int m) { return runs[m].cand_begin; };
  float acc[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) acc[k] = 0.f;
  if (c < st.cand_end) {
    const ScoreRun& ru = runs[last_at_most(st.run_begin, st.run_end, c, run_key)];
    const int page = ru.first_page + (c - ru.cand_begin);
    const int n_valid = min(P, ru.req_len - page * P);
    const int64_t phys = static_cast<int64_t>(ru.phys_base) + (c - ru.cand_begin);
    const int rows_q = P / kWarpsPerPage;
    const int r0 = qr * rows_q, r1 = min(n_valid, r0 + rows_q);
    const __nv_bfloat16* base = k_store + (phys * P) * D + lane * CPL;
#pragma unroll 4
    for (int r = r0; r < r1; ++r) {
      const __nv_bfloat16* kr = base + static_cast<int64_t>(r) * D;
      if constexpr (CPL == 4) {
        const uint2 raw = *reinterpret_cast<const uint2*>(kr);
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        acc[0] += x.x;
        acc[1] += x.y;
        acc[2] += y.x;
        acc[3] += y.y;
      } else {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kr));
        acc[0] += x.x;
        acc[1] += x.y;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < CPL; ++k) red[warp][lane * CPL + k] = acc[k];
  __syncthreads();
  for (int idx = threadIdx.x; idx < kScorePagesPerUnit * D; idx += kScoreThreads) {
    const int cc = idx / D, col = idx % D, cand = c0 + cc;
    if (cand >= st.cand_end) continue;
    const ScoreRun& ru = runs[last_at_most(st.run_begin, st.run_end, cand, run_key)];
    const int page = ru.first_page + (cand - ru.cand_begin);
    const int n_valid = min(P, ru.req_len - page * P);
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < kWarpsPerPage; ++w) t += red[cc * kWarpsPerPage + w][col];
    kbar[static_cast<int64_t>(cand) * D + col] = t / static_cast<float>(n_valid);
  }
}

// Ranks one table whose units are all done (their writes are visible: each
// unit ended with a fence before its counter bump).  Chunk sums and key
// means are read through L2 (ld.global.cg): other CTAs wrote them.
template <int D>
__device__ void rank_table(const ScoreView* sv, const ScoreTable& st, const ScoreFreqs& freqs,
                           const float* partials, const float* kbar, float* urot,
                           int32_t* out_pages, int32_t* out_count, float* out_scores,
                           int64_t scores_stride, uint8_t* smem) {
  using SM = ScoreSmem<D>;
  constexpr int H = D / 2, R = kScoreThreads / D, CPL = D / 32;
  unsigned long long* s_key = reinterpret_cast<unsigned long long*>(smem + SM::kOffKey);
  int* s_picked = reinterpret_cast<int*>(smem + SM::kOffPicked);
  float* u = reinterpret_cast<float*>(smem + SM::kOffU);
  float(*red)[D] = reinterpret_cast<float(*)[D]>(smem + SM::kOffRed);
  const ScoreRun* runs = reinterpret_cast<const ScoreRun*>(sv_arr(sv, sv->off_runs));
  auto run_key = [&](int m) { return runs[m].cand_begin; };
  const int t = st.table, top_k = sv->top_k;
  if (out_scores)
    for (int64_t c = threadIdx.x; c < scores_stride; c += kScoreThreads)
      out_scores[t * scores_stride + c] = __int_as_float(0x7fc00000);  // NaN
  // u: column c, chunks j, j + R, ... per thread, added in order, over the rows
  {
    const int c = threadIdx.x % D, j = threadIdx.x / D;
    float a = 0.f;
    for (int k = st.chunk_begin + j; k < st.chunk_end; k += R)
      a += __ldcg(partials + static_cast<int64_t>(k) * D + c);
    red[j][c] = a;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float tot = 0.f;
    for (int r = 0; r < R; ++r) tot += red[r][threadIdx.x];
    u[threadIdx.x] = tot / static_cast<float>(st.n_rows);
  }
  const int n = st.cand_end - st.cand_begin;
  int n2 = 1;
  while (n2 < n) n2 <<= 1;
  for (int x = n + threadIdx.x; x < n2; x += kScoreThreads) s_key[x] = 0;  // padding sorts last
  __syncthreads();
  // R(-delta) u of every run: u'_m = u_m cos + u_{m+H} sin, u'_{m+H} =
  // u_{m+H} cos - u_m sin (angle delta * f_m reduced mod 2 pi in fp64 with
  // 2 pi split in a head and a tail constant, sin / cos in fp32)
  const int n_run = st.run_end - st.run_begin;
  for (int e = threadIdx.x; e < n_run * H; e += kScoreThreads) {
    const int rn = st.run_begin + e / H, m = e % H;
    const int delta = runs[rn].delta;
    float sn = 0.f, cs = 1.f;
    if (delta != 0) {
      const double a = static_cast<double>(delta) * freqs.f[m];
      const double k2 = rint(a * 0.15915494309189535);
      double r2 = fma(-k2, 6.283185307179586, a);
      r2 = fma(-k2, 2.4492935982947064e-16, r2);
      sincosf(static_cast<float>(r2), &sn, &cs);
    }
    urot[static_cast<int64_t>(rn) * D + m] = u[m] * cs + u[m + H] * sn;
    urot[static_cast<int64_t>(rn) * D + m + H] = u[m + H] * cs - u[m] * sn;
  }
  __syncthreads();
  // one warp per candidate: lane l takes columns l * CPL .. of the key mean
  // and of its run's rotated u
  {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int x0 = warp * kRankBatch; x0 < n; x0 += kScoreWarps * kRankBatch) {
      float sc[kRankBatch];
#pragma unroll
      for (int b = 0; b < kRankBatch; ++b) {
        sc[b] = 0.f;
        const int x = x0 + b;
        if (x < n) {
          const int xc = st.cand_begin + x;
          const int rn = last_at_most(st.run_begin, st.run_end, xc, run_key);
          const float* kb = kbar + static_cast<int64_t>(xc) * D + lane * CPL;
          const float* ub = urot + static_cast<int64_t>(rn) * D + lane * CPL;
#pragma unroll
          for (int k = 0; k < CPL; ++k) sc[b] = fmaf(ub[k], __ldcg(kb + k), sc[b]);
        }
      }
#pragma unroll
      for (int b = 0; b < kRankBatch; ++b)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sc[b] += __shfl_xor_sync(0xffffffffu, sc[b], o);
      if (lane < kRankBatch && x0 + lane < n) {
        float mine = sc[0];
#pragma unroll
        for (int b = 1; b < kRankBatch; ++b) mine = lane == b ? sc[b] : mine;
        const int x = x0 + lane, xc = st.cand_begin + x;
        const ScoreRun& ru = runs[last_at_most(st.run_begin, st.run_end, xc, run_key)];
        const int pg = ru.first_page + (xc - ru.cand_begin);
        if (out_scores && pg < scores_stride) out_scores[t * scores_stride + pg] = mine;
        const float rank_sc = isnan(mine) ? -INFINITY : mine;  // a NaN score (bad input) ranks last
        s_key[x] = (static_cast<unsigned long long>(order_bits(rank_sc)) << 32) |
                   static_cast<uint32_t>(~static_cast<uint32_t>(pg));
      }
    }
  }
  __syncthreads();
  const int n_pick = n < top_k ? n : top_k;
  if (n <= kRankCount) {
    // rank of a key = the keys above it (keys are distinct: the page is in
    // the low bits); a candidate is picked if its rank is below n_pick, and
    // its output slot is the number of picked candidates before it (the
    // candidates ascend in page)
    for (int x = threadIdx.x; x < n; x += kScoreThreads) {
      const unsigned long long kx = s_key[x];
      int rank = 0;
      for (int y = 0; y < n; ++y) rank += s_key[y] > kx ? 1 : 0;
      s_picked[x] = rank < n_pick ? 1 : 0;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < n; x += kScoreThreads) {
      if (!s_picked[x]) continue;
      int pos = 0;
      for (int y = 0; y < x; ++y) pos += s_picked[y];
      out_pages[t * top_k + pos] = static_cast<int32_t>(~static_cast<uint32_t>(s_key[x]));
    }
  } else {
    // bitonic sort, descending: higher score first, equal score to the lower page
    for (int k = 2; k <= n2; k <<= 1)
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = threadIdx.x; i < n2; i += kScoreThreads) {
          const int p = i ^ j;
          if (p > i) {
            const unsigned long long a = s_key[i], b = s_key[p];
            if (((i & k) == 0) ? (a < b) : (a > b)) {
              s_key[i] = b;
              s_key[p] = a;
            }
          }
        }
        __syncthreads();
      }
    if (threadIdx.x < n_pick) {
      const uint32_t pg = ~static_cast<uint32_t>(s_key[threadIdx.x]);
      int pos = 0;
      for (int x = 0; x < n_pick; ++x) pos += (~static_cast<uint32_t>(s_key[x])) < pg ? 1 : 0;
      out_pages[t * top_k + pos] = static_cast<int32_t>(pg);
    }
  }
  if (threadIdx.x == 0) out_count[t] = n_pick;
}

template <int D>
__global__ void __launch_bounds__(kScoreThreads)
    score_kernel(const ScoreView* __restrict__ sv, const ScoreFreqs freqs,
                 const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k_store,
                 int P, float* partials, float* kbar, float* urot, int32_t* out_pages,
                 int32_t* out_count, float* out_scores, int64_t scores_stride) {
  extern __shared__ __align__(16) uint8_t score_smem[];
  __shared__ int s_last;
  const ScoreTable* tabs = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables));
  const ScoreRun* runs = reinterpret_cast<const ScoreRun*>(sv_arr(sv, sv->off_runs));
  const int32_t* table_map = sv_arr(sv, sv->off_table_map);
  int* done = const_cast<int*>(sv_arr(sv, sv->off_done));  // zeros in the uploaded image
  // tables of other classes (or without rows) pick nothing
  for (int t = blockIdx.x * kScoreThreads + threadIdx.x; t < sv->n_tables;
       t += gridDim.x * kScoreThreads) {
    if (table_map[t] >= 0) continue;
    out_count[t] = 0;
    if (out_scores)
      for (int64_t c = 0; c < scores_stride; ++c)
        out_scores[t * scores_stride + c] = __int_as_float(0x7fc00000);
  }
  const int n_chunks = sv->n_chunks, n_units = n_chunks + sv->n_page_units;
  for (int un = blockIdx.x; un < n_units; un += gridDim.x) {
    int st_idx;
    if (un < n_chunks) {
      st_idx = last_at_most(0, sv->n_st, un, [&](int m) { return tabs[m].chunk_begin; });
      query_unit<D>(sv, tabs[st_idx], un, q, partials, score_smem);
    } else {
      const int pu = un - n_chunks;
      st_idx = last_at_most(0, sv->n_st, pu, [&](int m) { return tabs[m].unit_begin; });
      const ScoreTable& st = tabs[st_idx];
      page_unit<D>(st, runs, st.cand_begin + (pu - st.unit_begin) * kScorePagesPerUnit, k_store,
                   P, kbar, score_smem);
    }
    __syncthreads();  // the unit's results are written; its shared memory is free
    if (threadIdx.x == 0) {
      __threadfence();
      const ScoreTable& st = tabs[st_idx];
      const int need = (st.chunk_end - st.chunk_begin) + (st.unit_end - st.unit_begin);
      s_last = atomicAdd(&done[st_idx], 1) == need - 1;
      if (s_last) __threadfence();
    }
    __syncthreads();
    if (s_last)
      rank_table<D>(sv, tabs[st_idx], freqs, partials, kbar, urot, out_pages, out_count,
                    out_scores, scores_stride, score_smem);
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_score(const ScoreView* sv_dev, const ScoreView& sv_host, const void* q,
                         const void* k_store, int D, int P, const double* inv_freq_host,
                         float* partials, float* kbar, float* urot, int32_t* out_pages,
                         int32_t* out_count, float* out_scores, int64_t scores_stride,
                         cudaStream_t stream) {
  ScoreFreqs f{};
  for (int m = 0; m < D / 2; ++m) f.f[m] = inv_freq_host[m];
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k_store);
  const int n_units = sv_host.n_chunks + sv_host.n_page_units;
  cudaError_t e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  // enough CTAs to fill the SMs (three resident per SM), at least one to
  // write the counts of a layout without retrieval work
  const int want = 3 * sms;
  const int grid = n_units > 0 ? (n_units < want ? n_units : want) : 1;
  auto launch = [&](auto kern, int smem) {
    cudaError_t r = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (r != cudaSuccess) return r;
    kern<<<grid, kScoreThreads, smem, stream>>>(sv_dev, f, qb, kb, P, partials, kbar, urot, out_pages,
                                                out_count, out_scores, scores_stride);
    return cudaGetLastError();
  };
  if (D == 128) return launch(score_kernel<128>, ScoreSmem<128>::kBytes);
  return launch(score_kernel<64>, ScoreSmem<64>::kBytes);
}

}  // namespace rk
