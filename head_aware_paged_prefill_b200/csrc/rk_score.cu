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
// segment that start at or before the last row) and its query chunks by
// the request's uncached row ranges; the kernels expand both.
// Two launches:
//   1. streaming (HBM bound): the first CTAs each sum the queries of a
//      64-row chunk of one table over the kv head's q heads (fp32, fixed
//      order, 16-byte loads); the others average the stored keys of 8
//      candidate pages, one warp per page;
//   2. one CTA per table: u from the table's chunk sums (in chunk order),
//      R(-delta) u of every run (into the workspace), one warp per candidate
//      for its dot product, then the picks: each candidate's rank is the
//      number of (score, page) keys above its own (up to 2048 candidates;
//      a bitonic sort in shared memory above that); the first k, in
//      ascending page order.
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

constexpr int kStreamThreads = 256;
static_assert(kStreamThreads == 32 * kScorePagesPerCta, "one warp per page");

// 1. query chunk sums and candidate key means.
//    Query CTA: thread (slot, column group) adds 8 consecutive columns (one
//    16-byte load) of the (row, head) pairs slot, slot + S, ...; the slots
//    are added in order.  Page CTA: warp w averages candidate 8 b + w, each
//    lane 128 / 32 = 4 columns (2 at D 64) of every key row.
template <int D>
__global__ void __launch_bounds__(kStreamThreads)
    score_stream_kernel(const ScoreView* __restrict__ sv, const __nv_bfloat16* __restrict__ q,
                        const __nv_bfloat16* __restrict__ k_store, int P,
                        float* __restrict__ partials, float* __restrict__ kbar) {
  constexpr int CG = D / 8;              // column groups of a query row
  constexpr int S = kStreamThreads / CG;  // query slots
  constexpr int CPL = D / 32;            // key columns per lane
  __shared__ float acc_s[S][D];
  const int n_chunks = sv->n_chunks;
  if (static_cast<int>(blockIdx.x) < n_chunks) {
    const ScoreTable* tabs = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables));
    const ScoreRange* rgs = reinterpret_cast<const ScoreRange*>(sv_arr(sv, sv->off_ranges));
    const int b = blockIdx.x;
    int lo = 0, hi = sv->n_st;  // last table with chunk_begin <= b
    while (hi - lo > 1) {
      const int m = (lo + hi) >> 1;
      if (tabs[m].chunk_begin <= b) lo = m; else hi = m;
    }
    const ScoreTable st = tabs[lo];
    int lc = b - st.chunk_begin, row_begin = 0, n_rows = 0;
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
      const uint4 raw =
          *reinterpret_cast<const uint4*>(q + (row * hq + st.head0 + h) * D + cg * 8);
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
    for (int c = threadIdx.x; c < D; c += kStreamThreads) {
      float t = 0.f;
      for (int sl = 0; sl < S; ++sl) t += acc_s[sl][c];
      partials[static_cast<int64_t>(blockIdx.x) * D + c] = t;
    }
    return;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cand = (blockIdx.x - n_chunks) * kScorePagesPerCta + warp;
  if (cand >= sv->n_cand) return;
  const ScoreRun* runs = reinterpret_cast<const ScoreRun*>(sv_arr(sv, sv->off_runs));
  int lo = 0, hi = sv->n_runs;  // last run with cand_begin <= cand
  while (hi - lo > 1) {
    const int m = (lo + hi) >> 1;
    if (runs[m].cand_begin <= cand) lo = m; else hi = m;
  }
  const ScoreRun rn = runs[lo];
  const int page = rn.first_page + (cand - rn.cand_begin);
  const int n_valid = min(P, rn.req_len - page * P);
  const int64_t phys = static_cast<int64_t>(rn.phys_base) + (cand - rn.cand_begin);
  const __nv_bfloat16* base = k_store + (phys * P) * D + lane * CPL;
  float acc[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) acc[k] = 0.f;
#pragma unroll 8
  for (int r = 0; r < n_valid; ++r) {
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
  const float inv = 1.f / static_cast<float>(n_valid);
#pragma unroll
  for (int k = 0; k < CPL; ++k)
    kbar[static_cast<int64_t>(cand) * D + lane * CPL + k] = acc[k] * inv;
}

__device__ __forceinline__ uint32_t order_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

constexpr int kRankThreads = 1024;
constexpr int kRankCount = 2048;  // candidates ranked by counting (a sort above)
constexpr int kRankBatch = 8;  // candidates a warp loads before reducing

// 2. scores and picks of one table
template <int D>
__global__ void __launch_bounds__(kRankThreads)
    score_rank_kernel(const ScoreView* __restrict__ sv, const ScoreFreqs freqs,
                      const float* __restrict__ partials, const float* __restrict__ kbar,
                      float* __restrict__ urot, int32_t* __restrict__ out_pages,
                      int32_t* __restrict__ out_count,
                      float* __restrict__ out_scores, int64_t scores_stride) {
  constexpr int H = D / 2;
  constexpr int R = kRankThreads / D;  // partial-sum runs per column
  extern __shared__ __align__(16) uint8_t rank_smem[];
  unsigned long long* s_key = reinterpret_cast<unsigned long long*>(rank_smem);  // [kScoreMaxCand]
  uint16_t* s_run = reinterpret_cast<uint16_t*>(s_key + kScoreMaxCand);         // [kScoreMaxCand]
  int* s_picked = reinterpret_cast<int*>(s_run + kScoreMaxCand);                 // [kRankCount]
  float* u = reinterpret_cast<float*>(s_picked + kRankCount);                    // [D]
  float(*red)[D] = reinterpret_cast<float(*)[D]>(u + D);                         // [R][D]
  const int t = blockIdx.x;
  const int top_k = sv->top_k;
  const int st_idx = sv_arr(sv, sv->off_table_map)[t];
  if (out_scores)
    for (int64_t c = threadIdx.x; c < scores_stride; c += kRankThreads)
      out_scores[t * scores_stride + c] = __int_as_float(0x7fc00000);  // NaN
  if (st_idx < 0) {
    if (threadIdx.x == 0) out_count[t] = 0;
    return;
  }
  const ScoreTable st = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables))[st_idx];
  const ScoreRun* runs = reinterpret_cast<const ScoreRun*>(sv_arr(sv, sv->off_runs));
  // u: the table's chunk sums, column c, chunks j, j + R, ... per thread,
  // runs added in order, divided by the row count
  {
    const int c = threadIdx.x % D, j = threadIdx.x / D;
    float a = 0.f;
#pragma unroll 8
    for (int k = st.chunk_begin + j; k < st.chunk_end; k += R)
      a += partials[static_cast<int64_t>(k) * D + c];
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
  for (int x = n + threadIdx.x; x < n2; x += kRankThreads) s_key[x] = 0;  // padding sorts last
  __syncthreads();
  // candidate -> run of the table (local index), for the dot products below
  for (int rn = st.run_begin; rn < st.run_end; ++rn)
    for (int x = runs[rn].cand_begin - st.cand_begin + threadIdx.x; x < runs[rn].cand_end - st.cand_begin;
         x += kRankThreads)
      s_run[x] = static_cast<uint16_t>(rn - st.run_begin);
  // R(-delta) u of every run of the table: u'_m = u_m cos + u_{m+H} sin,
  // u'_{m+H} = u_{m+H} cos - u_m sin (angle delta * f_m reduced mod 2 pi in
  // fp64 with 2 pi split in a head and a tail constant, sin / cos in fp32)
  const int n_run = st.run_end - st.run_begin;
  for (int e = threadIdx.x; e < n_run * H; e += kRankThreads) {
    const int rn = st.run_begin + e / H, m = e % H;
    const int delta = runs[rn].delta;
    float sn = 0.f, cs = 1.f;
    if (delta != 0) {
      const double a = static_cast<double>(delta) * freqs.f[m];
      const double n2pi = rint(a * 0.15915494309189535);
      double red2 = fma(-n2pi, 6.283185307179586, a);
      red2 = fma(-n2pi, 2.4492935982947064e-16, red2);
      sincosf(static_cast<float>(red2), &sn, &cs);
    }
    urot[static_cast<int64_t>(rn) * D + m] = u[m] * cs + u[m + H] * sn;
    urot[static_cast<int64_t>(rn) * D + m + H] = u[m + H] * cs - u[m] * sn;
  }
  __syncthreads();
  // one warp per candidate: lane l takes columns l * CPL .. + CPL - 1 of the
  // key mean and of its run's rotated u
  {
    constexpr int CPL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int NW = kRankThreads / 32;
    // run of a table-local candidate, from the map built above
    auto run_of = [&](int xc) { return st.run_begin + s_run[xc - st.cand_begin]; };
    for (int x0 = warp * kRankBatch; x0 < n; x0 += NW * kRankBatch) {
      float sc[kRankBatch];
#pragma unroll
      for (int b = 0; b < kRankBatch; ++b) {
        sc[b] = 0.f;
        const int x = x0 + b;
        if (x < n) {
          const int xc = st.cand_begin + x;
          const float* kb = kbar + static_cast<int64_t>(xc) * D + lane * CPL;
          const float* ub = urot + static_cast<int64_t>(run_of(xc)) * D + lane * CPL;
#pragma unroll
          for (int k = 0; k < CPL; ++k) sc[b] = fmaf(ub[k], kb[k], sc[b]);
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
        const ScoreRun& rn = runs[run_of(xc)];
        const int pg = rn.first_page + (xc - rn.cand_begin);
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
    for (int x = threadIdx.x; x < n; x += kRankThreads) {
      const unsigned long long kx = s_key[x];
      int rank = 0;
      for (int y = 0; y < n; ++y) rank += s_key[y] > kx ? 1 : 0;
      s_picked[x] = rank < n_pick ? 1 : 0;
    }
    __syncthreads();
    for (int x = threadIdx.x; x < n; x += kRankThreads) {
      if (!s_picked[x]) continue;
      int pos = 0;
      for (int y = 0; y < x; ++y) pos += s_picked[y];
      out_pages[t * top_k + pos] = static_cast<int32_t>(~static_cast<uint32_t>(s_key[x]));
    }
  } else {
    // bitonic sort, descending: higher score first, equal score to the lower page
    for (int k = 2; k <= n2; k <<= 1)
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = threadIdx.x; i < n2; i += kRankThreads) {
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
  const int n_stream = sv_host.n_chunks + sv_host.n_page_blocks;
  if (n_stream > 0) {
    if (D == 128)
      score_stream_kernel<128><<<n_stream, kStreamThreads, 0, stream>>>(sv_dev, qb, kb, P, partials, kbar);
    else
      score_stream_kernel<64><<<n_stream, kStreamThreads, 0, stream>>>(sv_dev, qb, kb, P, partials, kbar);
  }
  if (sv_host.n_tables > 0) {
    auto rank = [&](auto kern, int d) {
      const int smem = kScoreMaxCand * 10 + kRankCount * 4 + d * 4 + kRankThreads * 4;
      cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
      if (e != cudaSuccess) return e;
      kern<<<sv_host.n_tables, kRankThreads, smem, stream>>>(sv_dev, f, partials, kbar, urot,
                                                             out_pages, out_count, out_scores,
                                                             scores_stride);
      return cudaGetLastError();
    };
    return D == 128 ? rank(score_rank_kernel<128>, 128) : rank(score_rank_kernel<64>, 64);
  }
  return cudaGetLastError();
}

}  // namespace rk
