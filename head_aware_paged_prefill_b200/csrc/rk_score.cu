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
//            = mean over the page's keys of <R(-delta) u, K_stored>,
//              so u is rotated once per page instead of every key;
//   picks    = the top k candidate pages (cached, starting at or before the
//              last row), ties to the lower page, ascending page order.
//
// Three launches, all HBM-streaming:
//   1. one CTA per 64-row chunk of a table's rows sums those rows' queries
//      over the kv head's q heads (fp32, fixed order) into a partial;
//   2. one CTA per 8 candidate pages of one table adds the table's partials
//      in chunk order into u, then one warp per page streams the page once
//      (each lane 4 columns of every key row) against R(-delta) u;
//   3. one CTA per table selects the top k by repeated block arg-max (ties to
//      the lower page) and writes the picks, their count and the scores.
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

// 1. query partial sums: thread c2 owns columns 2 c2 and 2 c2 + 1
template <int D>
__global__ void __launch_bounds__(D / 2)
    score_query_kernel(const ScoreView* __restrict__ sv, const __nv_bfloat16* __restrict__ q,
                       float* __restrict__ partials) {
  const ScoreChunk ch = reinterpret_cast<const ScoreChunk*>(sv_arr(sv, sv->off_chunks))[blockIdx.x];
  const ScoreTable st = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables))[ch.st];
  const int g = sv->g, hq = sv->hq;
  const int c2 = threadIdx.x;
  float ax = 0.f, ay = 0.f;
  for (int i = 0; i < ch.n_rows; ++i) {
    const int64_t row = static_cast<int64_t>(st.q_row0) + ch.row_begin + i;
    const __nv_bfloat162* qr =
        reinterpret_cast<const __nv_bfloat162*>(q + (row * hq + st.head0) * D) + c2;
    for (int h = 0; h < g; ++h) {
      const float2 v = __bfloat1622float2(qr[h * (D / 2)]);
      ax += v.x;
      ay += v.y;
    }
  }
  partials[static_cast<int64_t>(blockIdx.x) * D + 2 * c2] = ax;
  partials[static_cast<int64_t>(blockIdx.x) * D + 2 * c2 + 1] = ay;
}

// 2. page scores: warp w of the CTA scores candidate first + w
template <int D>
__global__ void __launch_bounds__(32 * kScorePagesPerCta)
    score_pages_kernel(const ScoreView* __restrict__ sv, const __nv_bfloat16* __restrict__ k_store,
                       int P, const ScoreFreqs freqs, const float* __restrict__ partials,
                       float* __restrict__ cand_scores) {
  constexpr int H = D / 2;
  constexpr int CPL = D / 32;  // columns per lane: 4 (D 128) or 2 (D 64)
  __shared__ float u[D];
  const int2 blk = reinterpret_cast<const int2*>(sv_arr(sv, sv->off_blocks))[blockIdx.x];
  const ScoreTable st = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables))[blk.x];
  for (int c = threadIdx.x; c < D; c += blockDim.x) {
    float acc = 0.f;
    for (int k = st.chunk_begin; k < st.chunk_end; ++k) acc += partials[static_cast<int64_t>(k) * D + c];
    u[c] = acc / static_cast<float>(st.n_rows);
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cand = blk.y + warp;
  if (cand >= st.cand_end) return;
  const ScoreCand cd = reinterpret_cast<const ScoreCand*>(sv_arr(sv, sv->off_cand))[cand];
  // this lane's columns of R(-delta) u: u'_m = u_m cos + u_{m+H} sin,
  // u'_{m+H} = u_{m+H} cos - u_m sin (angle delta * f_m, reduced mod 2 pi in
  // fp64 with 2 pi split in a head and a tail constant, sin / cos in fp32)
  float w[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) {
    const int c = lane * CPL + k;
    const int m = c < H ? c : c - H;
    float sn = 0.f, cs = 1.f;
    if (cd.delta != 0) {
      const double a = static_cast<double>(cd.delta) * freqs.f[m];
      const double n2pi = rint(a * 0.15915494309189535);
      double red = fma(-n2pi, 6.283185307179586, a);
      red = fma(-n2pi, 2.4492935982947064e-16, red);
      sincosf(static_cast<float>(red), &sn, &cs);
    }
    w[k] = c < H ? u[c] * cs + u[c + H] * sn : u[c] * cs - u[c - H] * sn;
  }
  const __nv_bfloat16* base = k_store + (static_cast<int64_t>(cd.phys) * P) * D + lane * CPL;
  float acc = 0.f;
#pragma unroll 8
  for (int r = 0; r < cd.n_valid; ++r) {
    const __nv_bfloat16* kr = base + static_cast<int64_t>(r) * D;
    if constexpr (CPL == 4) {
      const uint2 raw = *reinterpret_cast<const uint2*>(kr);
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
      const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
      acc = fmaf(w[0], a.x, acc);
      acc = fmaf(w[1], a.y, acc);
      acc = fmaf(w[2], b.x, acc);
      acc = fmaf(w[3], b.y, acc);
    } else {
      const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kr));
      acc = fmaf(w[0], a.x, acc);
      acc = fmaf(w[1], a.y, acc);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) cand_scores[cand] = acc / static_cast<float>(cd.n_valid);
}

constexpr int kTopkThreads = 256;

// 3. top k of one table
__global__ void __launch_bounds__(kTopkThreads)
    score_topk_kernel(const ScoreView* __restrict__ sv, const float* __restrict__ cand_scores,
                      int32_t* __restrict__ out_pages, int32_t* __restrict__ out_count,
                      float* __restrict__ out_scores, int64_t scores_stride) {
  __shared__ float s_score[kScoreMaxCand];
  __shared__ int s_page[kScoreMaxCand];
  __shared__ float red_s[kTopkThreads / 32];
  __shared__ int red_i[kTopkThreads / 32];
  __shared__ int picks[kScoreMaxTopK];
  const int t = blockIdx.x;
  const int top_k = sv->top_k;
  const int st_idx = sv_arr(sv, sv->off_table_map)[t];
  if (out_scores)
    for (int64_t c = threadIdx.x; c < scores_stride; c += kTopkThreads)
      out_scores[t * scores_stride + c] = __int_as_float(0x7fc00000);  // NaN
  if (st_idx < 0) {
    if (threadIdx.x == 0) out_count[t] = 0;
    return;
  }
  const ScoreTable st = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables))[st_idx];
  const ScoreCand* cands = reinterpret_cast<const ScoreCand*>(sv_arr(sv, sv->off_cand));
  const int n = st.cand_end - st.cand_begin;
  __syncthreads();  // the NaN fill precedes the candidates' scores
  for (int x = threadIdx.x; x < n; x += kTopkThreads) {
    const float sc = cand_scores[st.cand_begin + x];
    const int pg = cands[st.cand_begin + x].page;
    s_score[x] = isnan(sc) ? -INFINITY : sc;  // a NaN score (bad input) ranks last
    s_page[x] = pg;
    if (out_scores && pg < scores_stride) out_scores[t * scores_stride + pg] = sc;
  }
  __syncthreads();
  const int n_pick = n < top_k ? n : top_k;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int k = 0; k < n_pick; ++k) {
    // best remaining candidate: highest score, then lowest page (a taken
    // candidate carries score -inf and page INT_MAX)
    float bs = -INFINITY;
    int bp = 0x7fffffff, bx = -1;
    for (int x = threadIdx.x; x < n; x += kTopkThreads) {
      const float sc = s_score[x];
      const int pg = s_page[x];
      if (sc > bs || (sc == bs && pg < bp)) {
        bs = sc;
        bp = pg;
        bx = x;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float os = __shfl_xor_sync(0xffffffffu, bs, o);
      const int op = __shfl_xor_sync(0xffffffffu, bp, o);
      const int ox = __shfl_xor_sync(0xffffffffu, bx, o);
      if (os > bs || (os == bs && op < bp)) {
        bs = os;
        bp = op;
        bx = ox;
      }
    }
    if (lane == 0) {
      red_s[warp] = bs;
      red_i[warp] = bx;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      float b = -INFINITY;
      int bi = -1, bpg = 0x7fffffff;
      for (int w = 0; w < kTopkThreads / 32; ++w) {
        const int xi = red_i[w];
        if (xi < 0) continue;
        const int pg = s_page[xi];
        if (red_s[w] > b || (red_s[w] == b && pg < bpg)) {
          b = red_s[w];
          bi = xi;
          bpg = pg;
        }
      }
      picks[k] = bpg;
      if (bi >= 0) {
        s_score[bi] = -INFINITY;
        s_page[bi] = 0x7fffffff;
      }
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    // ascending page order (n_pick <= 64)
    for (int a = 1; a < n_pick; ++a) {
      const int v = picks[a];
      int b = a - 1;
      while (b >= 0 && picks[b] > v) {
        picks[b + 1] = picks[b];
        --b;
      }
      picks[b + 1] = v;
    }
    out_count[t] = n_pick;
  }
  __syncthreads();
  for (int k = threadIdx.x; k < n_pick; k += kTopkThreads) out_pages[t * top_k + k] = picks[k];
}

}  // namespace

cudaError_t launch_score(const ScoreView* sv_dev, const ScoreView& sv_host, const void* q,
                         const void* k_store, int D, int P, const double* inv_freq_host,
                         float* partials, float* cand_scores, int32_t* out_pages,
                         int32_t* out_count, float* out_scores, int64_t scores_stride,
                         cudaStream_t stream) {
  ScoreFreqs f{};
  for (int m = 0; m < D / 2; ++m) f.f[m] = inv_freq_host[m];
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k_store);
  if (sv_host.n_chunks > 0) {
    if (D == 128)
      score_query_kernel<128><<<sv_host.n_chunks, 64, 0, stream>>>(sv_dev, qb, partials);
    else
      score_query_kernel<64><<<sv_host.n_chunks, 32, 0, stream>>>(sv_dev, qb, partials);
  }
  if (sv_host.n_blocks > 0) {
    if (D == 128)
      score_pages_kernel<128><<<sv_host.n_blocks, 32 * kScorePagesPerCta, 0, stream>>>(
          sv_dev, kb, P, f, partials, cand_scores);
    else
      score_pages_kernel<64><<<sv_host.n_blocks, 32 * kScorePagesPerCta, 0, stream>>>(
          sv_dev, kb, P, f, partials, cand_scores);
  }
  if (sv_host.n_tables > 0)
    score_topk_kernel<<<sv_host.n_tables, kTopkThreads, 0, stream>>>(
        sv_dev, cand_scores, out_pages, out_count, out_scores, scores_stride);
  return cudaGetLastError();
}

}  // namespace rk
