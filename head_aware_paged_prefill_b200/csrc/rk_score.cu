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
// request's uncached ranges; the kernels expand both.  Three launches:
//   1. queries (HBM bound): one CTA per 64-row chunk of a table sums the
//      chunk's queries over the kv head's q heads (fp32, fixed order,
//      16-byte loads).  The CTA that finishes a table's last chunk (a
//      counter per table) adds the chunk sums in chunk order into u and
//      writes R(-delta) u for each of the table's runs;
//   2. pages (HBM bound): one warp per candidate page sums the page's
//      stored keys and takes the dot product of their mean with its run's
//      rotated u at once, so the page's score and its rank key leave the
//      launch;
//   3. picks, one CTA per table: the k largest (score, page) keys, found
//      by a radix select on the 64-bit key a byte at a time, written in
//      ascending page order by a block-wide scan.
// Launches 2 and 3 are programmatic dependents of the one before: the page
// launch starts while the query launch still streams and waits for it only
// before it reads the rotated u, and the pick launch waits before it reads
// the scores.
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

constexpr int kQueryThreads = 256;
constexpr int kPageThreads = 32 * kScorePagesPerCta;  // one warp per page
constexpr int kPickThreads = 1024;

// Programmatic dependent launch: let the next launch on the stream begin,
// and wait until the launch before has completed with its writes visible
// (a no-op when this launch was not made a dependent).
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint32_t order_bits(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// 1. query chunk sums; the last chunk of a table forms R(-delta) u per run.
// Thread (slot, column group) adds 8 consecutive columns (one 16-byte load)
// of the (row, head) pairs slot, slot + S, ...; the slots are added in order.
template <int D>
__global__ void __launch_bounds__(kQueryThreads)
    score_query_kernel(const ScoreView* __restrict__ sv, const ScoreFreqs freqs,
                       const __nv_bfloat16* __restrict__ q, float* partials, float* urot) {
  constexpr int CG = D / 8, S = kQueryThreads / CG, H = D / 2, R = kQueryThreads / D;
  __shared__ float acc_s[S][D];
  __shared__ float u[D];
  __shared__ int s_last;
  pdl_launch_dependents();  // the page launch streams its keys meanwhile
  const ScoreTable* tabs = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables));
  const ScoreRange* rgs = reinterpret_cast<const ScoreRange*>(sv_arr(sv, sv->off_ranges));
  const ScoreRun* runs = reinterpret_cast<const ScoreRun*>(sv_arr(sv, sv->off_runs));
  int* done = const_cast<int*>(sv_arr(sv, sv->off_done));  // zeros in the uploaded image
  const int b = blockIdx.x;
  const int st_idx = sv_arr(sv, sv->off_chunk_table)[b];
  const ScoreTable st = tabs[st_idx];
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
  for (int c = threadIdx.x; c < D; c += kQueryThreads) {
    float t = 0.f;
    for (int sl = 0; sl < S; ++sl) t += acc_s[sl][c];
    partials[static_cast<int64_t>(b) * D + c] = t;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    s_last = atomicAdd(&done[st_idx], 1) == st.chunk_end - st.chunk_begin - 1;
    if (s_last) __threadfence();
  }
  __syncthreads();
  if (!s_last) return;
  // u: column c, chunks j, j + R, ... per thread, added in order, over the rows
  {
    const int c = threadIdx.x % D, j = threadIdx.x / D;
    float t = 0.f;
    for (int k0 = st.chunk_begin + j; k0 < st.chunk_end; k0 += 8 * R) {
      float v[8];  // eight loads in flight, added in chunk order
#pragma unroll
      for (int x = 0; x < 8; ++x) {
        const int k = k0 + x * R;
        v[x] = k < st.chunk_end ? __ldcg(partials + static_cast<int64_t>(k) * D + c) : 0.f;
      }
#pragma unroll
      for (int x = 0; x < 8; ++x) t += v[x];
    }
    acc_s[j][c] = t;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    float tot = 0.f;
    for (int j = 0; j < R; ++j) tot += acc_s[j][threadIdx.x];
    u[threadIdx.x] = tot / static_cast<float>(st.n_rows);
  }
  __syncthreads();
  // R(-delta) u of every run: u'_m = u_m cos + u_{m+H} sin, u'_{m+H} =
  // u_{m+H} cos - u_m sin (angle delta * f_m reduced mod 2 pi in fp64 with
  // 2 pi split in a head and a tail constant, sin / cos in fp32)
  const int n_run = st.run_end - st.run_begin;
  for (int e = threadIdx.x; e < n_run * H; e += kQueryThreads) {
    const int rn = st.run_begin + e / H, m = e % H;
    const int delta = runs[rn].delta;
    float sn = 0.f, cs = 1.f;
    if (delta != 0) {
      const double ang = static_cast<double>(delta) * freqs.f[m];
      const double k2 = rint(ang * 0.15915494309189535);
      double r2 = fma(-k2, 6.283185307179586, ang);
      r2 = fma(-k2, 2.4492935982947064e-16, r2);
      sincosf(static_cast<float>(r2), &sn, &cs);
    }
    urot[static_cast<int64_t>(rn) * D + m] = u[m] * cs + u[m + H] * sn;
    urot[static_cast<int64_t>(rn) * D + m + H] = u[m + H] * cs - u[m] * sn;
  }
}

// 2. one warp per candidate page: the mean of its stored keys (lane l takes
// columns l * CPL ..) and its dot product with the run's rotated u
template <int D>
__global__ void __launch_bounds__(kPageThreads)
    score_page_kernel(const ScoreView* __restrict__ sv, const __nv_bfloat16* __restrict__ k_store,
                      int P, const float* __restrict__ urot, float* __restrict__ scores,
                      unsigned long long* __restrict__ keys) {
  constexpr int CPL = D / 32;
  pdl_launch_dependents();  // the pick launch waits for this one to complete
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cand = blockIdx.x * kScorePagesPerCta + warp;
  if (cand >= sv->n_cand) return;
  const ScoreRun* runs = reinterpret_cast<const ScoreRun*>(sv_arr(sv, sv->off_runs));
  // the run of the block's first candidate, then forward to this warp's
  int rn = sv_arr(sv, sv->off_block_run)[blockIdx.x];
  while (rn + 1 < sv->n_runs && runs[rn + 1].cand_begin <= cand) ++rn;
  const ScoreRun ru = runs[rn];
  const int page = ru.first_page + (cand - ru.cand_begin);
  const int n_valid = min(P, ru.req_len - page * P);
  const int64_t phys = static_cast<int64_t>(ru.phys_base) + (cand - ru.cand_begin);
  const __nv_bfloat16* base = k_store + (phys * P) * D + lane * CPL;
  float acc[CPL];
#pragma unroll
  for (int k = 0; k < CPL; ++k) acc[k] = 0.f;
  // rows in batches of 16 loads in flight (two rounds for a 64-key page),
  // added in row order
  for (int r0 = 0; r0 < n_valid; r0 += 16) {
    if constexpr (CPL == 4) {
      uint2 raw[16];
      if (r0 + 16 <= n_valid) {
#pragma unroll
        for (int x = 0; x < 16; ++x)
          raw[x] = *reinterpret_cast<const uint2*>(base + static_cast<int64_t>(r0 + x) * D);
      } else {
#pragma unroll
        for (int x = 0; x < 16; ++x)
          raw[x] = r0 + x < n_valid ? *reinterpret_cast<const uint2*>(base + static_cast<int64_t>(r0 + x) * D)
                                    : make_uint2(0u, 0u);
      }
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[x].x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[x].y));
        acc[0] += a.x;
        acc[1] += a.y;
        acc[2] += b.x;
        acc[3] += b.y;
      }
    } else {
      uint32_t raw[16];
      if (r0 + 16 <= n_valid) {
#pragma unroll
        for (int x = 0; x < 16; ++x)
          raw[x] = *reinterpret_cast<const uint32_t*>(base + static_cast<int64_t>(r0 + x) * D);
      } else {
#pragma unroll
        for (int x = 0; x < 16; ++x)
          raw[x] = r0 + x < n_valid ? *reinterpret_cast<const uint32_t*>(base + static_cast<int64_t>(r0 + x) * D)
                                    : 0u;
      }
#pragma unroll
      for (int x = 0; x < 16; ++x) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw[x]));
        acc[0] += a.x;
        acc[1] += a.y;
      }
    }
  }
  pdl_wait();  // the query launch's rotated u
  const float inv = 1.f / static_cast<float>(n_valid);
  const float* ub = urot + static_cast<int64_t>(rn) * D + lane * CPL;
  float sc = 0.f;
#pragma unroll
  for (int k = 0; k < CPL; ++k) sc = fmaf(ub[k], acc[k] * inv, sc);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sc += __shfl_xor_sync(0xffffffffu, sc, o);
  if (lane == 0) {
    scores[cand] = sc;
    const float rank_sc = isnan(sc) ? -INFINITY : sc;  // a NaN score (bad input) ranks last
    keys[cand] = (static_cast<unsigned long long>(order_bits(rank_sc)) << 32) |
                 static_cast<uint32_t>(~static_cast<uint32_t>(page));
  }
}

// 3. the picks of one table from its candidates' scores
__global__ void __launch_bounds__(kPickThreads)
    score_pick_kernel(const ScoreView* __restrict__ sv, const float* __restrict__ scores,
                      const unsigned long long* __restrict__ keys, int32_t* __restrict__ out_pages,
                      int32_t* __restrict__ out_count,
                      float* __restrict__ out_scores, int64_t scores_stride) {
  __shared__ unsigned long long s_key[kScoreMaxCand];
  __shared__ int s_hist[256];
  __shared__ int s_sel[3];
  __shared__ int s_warp[kPickThreads / 32];
  const int t = blockIdx.x;
  const int top_k = sv->top_k;
  const int st_idx = sv_arr(sv, sv->off_table_map)[t];
  if (out_scores)
    for (int64_t c = threadIdx.x; c < scores_stride; c += kPickThreads)
      out_scores[t * scores_stride + c] = __int_as_float(0x7fc00000);  // NaN
  // the plan (uploaded before the first launch) is read before the wait
  ScoreTable st{};
  if (st_idx >= 0) st = reinterpret_cast<const ScoreTable*>(sv_arr(sv, sv->off_tables))[st_idx];
  const int n = st_idx >= 0 ? st.cand_end - st.cand_begin : 0;
  pdl_wait();  // the page launch's scores and keys
  if (st_idx < 0) {
    if (threadIdx.x == 0) out_count[t] = 0;
    return;
  }
  if (out_scores) __syncthreads();  // the NaN fill lands before the scores
  for (int x = threadIdx.x; x < n; x += kPickThreads) {
    const unsigned long long key = keys[st.cand_begin + x];
    s_key[x] = key;
    const uint32_t pg = ~static_cast<uint32_t>(key);
    if (out_scores && pg < scores_stride) out_scores[t * scores_stride + pg] = scores[st.cand_begin + x];
  }
  __syncthreads();
  const int n_pick = n < top_k ? n : top_k;
  {
    // the picks are the n_pick largest keys (distinct: the page is in the
    // low bits), found by a radix select from the top byte down: prefix /
    // mask hold the decided high bits of the threshold, `need` the picks
    // still to take among keys matching them; a key is picked when its
    // decided bits reach the prefix.  The select stops as soon as the
    // keys matching the prefix are exactly the picks still needed.
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    unsigned long long prefix = 0ull, mask = 0ull;
    int need = n_pick;
    for (int shift = 56; shift >= 0 && need > 0; shift -= 8) {
      if (threadIdx.x < 256) s_hist[threadIdx.x] = 0;
      __syncthreads();
      for (int x = threadIdx.x; x < n; x += kPickThreads) {
        const unsigned long long kx = s_key[x];
        if ((kx & mask) == prefix) atomicAdd(&s_hist[(kx >> shift) & 255u], 1);
      }
      __syncthreads();
      if (w == 0) {
        // lane l holds digits 255 - 8l down to 248 - 8l (descending)
        int c[8], loc = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          c[j] = s_hist[255 - 8 * lane - j];
          loc += c[j];
        }
        int incl = loc;
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += u;
        }
        int above = incl - loc;  // keys matching the prefix with a larger digit
        if (above < need && need <= incl) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            if (above + c[j] >= need) {
              s_sel[0] = 255 - 8 * lane - j;
              s_sel[1] = above;
              s_sel[2] = c[j];
              break;
            }
            above += c[j];
          }
        }
      }
      __syncthreads();
      const int d = s_sel[0], above = s_sel[1], cnt = s_sel[2];
      prefix |= static_cast<unsigned long long>(d) << shift;
      mask |= 255ull << shift;
      need -= above;
      if (cnt == need) need = 0;  // every key matching the prefix is a pick
      __syncthreads();           // s_hist and s_sel are reused
    }
    // output slot = picked candidates before it (the candidates ascend in
    // page): ballots within a warp, the warps' counts scanned by warp 0
    int placed = 0;
    for (int base = 0; base < n; base += kPickThreads) {
      const int x = base + threadIdx.x;
      const bool f = x < n && (s_key[x] & mask) >= prefix;
      const unsigned m = __ballot_sync(0xffffffffu, f);
      if (lane == 0) s_warp[w] = __popc(m);
      __syncthreads();
      if (w == 0) {
        int v = s_warp[lane];
        for (int o = 1; o < 32; o <<= 1) {
          const int u = __shfl_up_sync(0xffffffffu, v, o);
          if (lane >= o) v += u;
        }
        s_warp[lane] = v;  // inclusive prefix over the warps
      }
      __syncthreads();
      if (f) {
        const int pos = placed + (w ? s_warp[w - 1] : 0) + __popc(m & ((1u << lane) - 1u));
        out_pages[t * top_k + pos] = static_cast<int32_t>(~static_cast<uint32_t>(s_key[x]));
      }
      placed += s_warp[kPickThreads / 32 - 1];
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) out_count[t] = n_pick;
}

}  // namespace

cudaError_t launch_score(const ScoreView* sv_dev, const ScoreView& sv_host, const void* q,
                         const void* k_store, int D, int P, const double* inv_freq_host,
                         float* partials, float* scores, float* urot, int32_t* out_pages,
                         int32_t* out_count, float* out_scores, int64_t scores_stride,
                         cudaStream_t stream) {
  ScoreFreqs f{};
  for (int m = 0; m < D / 2; ++m) f.f[m] = inv_freq_host[m];
  const auto* qb = static_cast<const __nv_bfloat16*>(q);
  const auto* kb = static_cast<const __nv_bfloat16*>(k_store);
  if (sv_host.n_chunks > 0) {
    if (D == 128)
      score_query_kernel<128><<<sv_host.n_chunks, kQueryThreads, 0, stream>>>(sv_dev, f, qb, partials, urot);
    else
      score_query_kernel<64><<<sv_host.n_chunks, kQueryThreads, 0, stream>>>(sv_dev, f, qb, partials, urot);
  }
  // the scores, then (8-byte aligned) the rank keys, share one workspace slot
  auto* keys = reinterpret_cast<unsigned long long*>(
      scores + ((static_cast<int64_t>(sv_host.n_cand) + 1) & ~static_cast<int64_t>(1)));
  cudaLaunchAttribute pdl[1];
  pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  pdl[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg{};
  cfg.stream = stream;
  cfg.attrs = pdl;
  cfg.numAttrs = 1;
  cudaError_t e = cudaSuccess;
  if (sv_host.n_page_blocks > 0) {
    cfg.gridDim = dim3(sv_host.n_page_blocks);
    cfg.blockDim = dim3(kPageThreads);
    e = D == 128 ? cudaLaunchKernelEx(&cfg, score_page_kernel<128>, sv_dev, kb, P,
                                      static_cast<const float*>(urot), scores, keys)
                 : cudaLaunchKernelEx(&cfg, score_page_kernel<64>, sv_dev, kb, P,
                                      static_cast<const float*>(urot), scores, keys);
    if (e != cudaSuccess) return e;
  }
  if (sv_host.n_tables > 0) {
    cfg.gridDim = dim3(sv_host.n_tables);
    cfg.blockDim = dim3(kPickThreads);
    e = cudaLaunchKernelEx(&cfg, score_pick_kernel, sv_dev, static_cast<const float*>(scores),
                           static_cast<const unsigned long long*>(keys), out_pages, out_count,
                           out_scores, scores_stride);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace rk
