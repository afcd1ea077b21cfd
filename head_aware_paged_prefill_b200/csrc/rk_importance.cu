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
// Three launches:
//   1. column sums, one CTA per (table, 128 keys).  Each warp holds two
//      16-key slices of relocated K in registers as the A operand of warp-level
//      bf16 MMAs; the CTA streams tiles of 64 (row, q head) columns of Q (and
//      their lse) through a three-deep cp.async ring, only the rows of the
//      table's row set that can see its keys (causal from its lowest key, up
//      to its highest key + W - 1 for local tables).  S = K Q^T, then
//      P = 2^(S scale log2 e - lse log2 e) masked per element, summed per key
//      in registers and over the four lanes of a key at the end.  A CTA
//      takes one chunk of 8192 / G rows (chunks aligned on row 0, so the
//      CTAs of a chunk read the same Q rows from L2 and no CTA walks a whole
//      long request); each (layer, kv head, chunk, token) partial is written
//      by exactly one CTA.
//   2. the partials added over kv heads and chunks in a fixed order: the
//      importance.
//   3. per (request, layer), one 1024-thread CTA: a four-pass radix select
//      on the float bits (all values are >= +0, so the bits order like the
//      values) finds the k-th value; ordered block scans then emit the
//      positions above it and the lowest positions equal to it, ascending.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <climits>
#include <cmath>
#include <cstdint>

#include "rk_internal.h"

namespace rk {

namespace {

constexpr int kImpThreads = 128;
constexpr int kImpWarps = kImpThreads / 32;
constexpr int kImpSlices = 2;  // 16-key slices per warp
constexpr int kImpCols = 64;   // (row, q head) columns per Q tile
constexpr int kImpStages = 3;  // Q tiles in flight per CTA
constexpr int kImpSelectThreads = 1024;
constexpr float kLog2e = 1.4426950408889634f;
static_assert(kImpWarps * kImpSlices * 16 == kImpKeysPerCta, "keys per CTA");

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
  const float* lse;
  float* part;
  float* importance;
  int32_t* tokens;
  int32_t* token_count;
  int64_t n_pages;
  int n_req, n_layers, hq, hkv, p, total_tokens, window, top_k, n_chunks;
  float scale_log2;
  int8_t cls[kImpMaxLh];
  int32_t* error_word;
};

__device__ __forceinline__ uint32_t shared_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(shared_addr(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(shared_addr(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Four 8x8 bf16 matrices from shared memory; lanes 8i..8i+7 address the rows
// of matrix i, and lane l receives row l / 4, columns 2 (l % 4) + {0, 1}.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

// 2^x on the special function unit (flushes results below 2^-126 to 0,
// which a sum of weights in [0, 1] does not notice)
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// c (16 x 8, fp32) += A (16 x 16, bf16) B (16 x 8, bf16)
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// A run of Q tile columns: flat (row, q head) indices [f0, fend), f = row G + h.
struct ColTile {
  int ri, f0, fend;
};

// 1. column sums of one table's 128 keys
template <int D, int G>
__global__ void __launch_bounds__(kImpThreads)
    importance_colsum_kernel(const __grid_constant__ ImpArgs a) {
  constexpr int KS = D / 16;
  constexpr int CHUNKS = D / 8;
  extern __shared__ __align__(128) uint8_t imp_smem[];
  // [kImpStages][kImpCols][D] Q columns, then [kImpStages][kImpCols] lse
  auto sQ = reinterpret_cast<__nv_bfloat16(*)[kImpCols * D]>(imp_smem);
  auto sL = reinterpret_cast<float(*)[kImpCols]>(imp_smem + kImpStages * kImpCols * D * 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;
  const int t = blockIdx.x;
  const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
  const int n_e = a.entry_count[t], e_first = a.entry_start[t], rc = a.range_count[t];
  const int spp = a.p / 16;
  const int n_sl = n_e * spp;
  const int s_begin = blockIdx.y * (kImpWarps * kImpSlices);
  if (s_begin >= n_sl || rc == 0) return;
  const int s_end = min(n_sl, s_begin + kImpWarps * kImpSlices);
  const int t0 = a.cu[r], L = a.cu[r + 1] - t0;
  const bool local = a.cls[layer * a.hkv + kvh] == RK_LOCAL;
  const int W = a.window;
  // the CTA's lowest and highest key positions (entries ascend)
  int pos_lo, pos_hi;
  {
    const rk_entry e0 = a.entries[e_first + s_begin / spp];
    pos_lo = e0.logical_pos + (s_begin % spp) * 16;
    const int sl = s_end - 1;
    const rk_entry e1 = a.entries[e_first + sl / spp];
    pos_hi = e1.logical_pos + min((sl % spp) * 16 + 16, e1.n_valid) - 1;
  }
  // rows that can see these keys (causal from the lowest; for a local table,
  // up to the highest + W - 1), cut to this CTA's chunk of kImpChunkCols / G
  // rows (chunks are aligned on row 0, so the CTAs of one chunk read the same
  // Q rows while they are in L2)
  constexpr int RPC = kImpChunkCols / G;
  const int chunk = blockIdx.z;
  const int row_lo = max(pos_lo, chunk * RPC);
  const int row_hi =
      min(local ? min(L - 1, pos_hi + min(W, L) - 1) : L - 1, chunk * RPC + RPC - 1);
  if (row_lo > row_hi) return;
  // this warp's keys as A fragments (a0: key gq, columns 2 tq; a1: key gq + 8;
  // a2, a3: columns + 8), and their positions (INT_MAX: no key)
  uint32_t ka[kImpSlices][KS][4];
  int kpos[kImpSlices][2];
#pragma unroll
  for (int u = 0; u < kImpSlices; ++u) {
    kpos[u][0] = kpos[u][1] = INT_MAX;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) ka[u][ks][0] = ka[u][ks][1] = ka[u][ks][2] = ka[u][ks][3] = 0u;
    const int s = s_begin + warp * kImpSlices + u;
    if (s >= s_end) continue;
    const rk_entry en = a.entries[e_first + s / spp];
    const int k0 = (s % spp) * 16;
    if (en.phys_page < 0 || en.phys_page >= a.n_pages) {
      if (lane == 0) atomicOr(a.error_word, static_cast<int>(RK_DEV_BAD_PAGE));
      continue;
    }
    const uint32_t* kr = reinterpret_cast<const uint32_t*>(
        a.k_pool + (static_cast<int64_t>(en.phys_page) * a.p + k0) * D);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      ka[u][ks][0] = kr[gq * (D / 2) + ks * 8 + tq];
      ka[u][ks][1] = kr[(gq + 8) * (D / 2) + ks * 8 + tq];
      ka[u][ks][2] = kr[gq * (D / 2) + ks * 8 + 4 + tq];
      ka[u][ks][3] = kr[(gq + 8) * (D / 2) + ks * 8 + 4 + tq];
    }
    if (k0 + gq < en.n_valid) kpos[u][0] = en.logical_pos + k0 + gq;
    if (k0 + gq + 8 < en.n_valid) kpos[u][1] = en.logical_pos + k0 + gq + 8;
  }
  // every key of the CTA is a real key (then a tile whose rows all see all
  // keys needs no per-element mask)
  const bool keys_full = __syncthreads_and(kpos[0][0] != INT_MAX && kpos[0][1] != INT_MAX &&
                                           kpos[1][0] != INT_MAX && kpos[1][1] != INT_MAX);
  // column tiles: the table's row ranges clipped to [row_lo, row_hi]
  const rk_range* rg = a.ranges + a.range_start[t];
  auto seek = [&](int ri, ColTile& it) -> bool {
    for (; ri < rc; ++ri) {
      const rk_range x = rg[ri];
      if (x.begin > row_hi) return false;
      const int b0 = max(x.begin, row_lo), b1 = min(x.end, row_hi + 1);
      if (b0 < b1) {
        it.ri = ri;
        it.f0 = b0 * G;
        it.fend = b1 * G;
        return true;
      }
    }
    return false;
  };
  auto advance = [&](ColTile& it) -> bool {
    it.f0 += kImpCols;
    if (it.f0 < it.fend) return true;
    return seek(it.ri + 1, it);
  };
  // stage a tile's Q columns (16-byte chunks permuted per column, chunk c of
  // column n at c ^ (n & 7)) and their lse, all by cp.async
  auto stage = [&](const ColTile& it, int buf) {
    for (int x = threadIdx.x; x < kImpCols * CHUNKS; x += kImpThreads) {
      const int n = x / CHUNKS, c = x % CHUNKS;
      const int f = it.f0 + n;
      if (f < it.fend) {
        const int i = f / G, h = f - i * G;
        const __nv_bfloat16* src =
            a.q + ((static_cast<int64_t>(layer) * a.total_tokens + t0 + i) * a.hq + kvh * G + h) * D +
            c * 8;
        cp_async16(&sQ[buf][n * D + (c ^ (n & 7)) * 8], src);
      }
    }
    if (threadIdx.x < kImpCols) {
      const int f = it.f0 + threadIdx.x;
      if (f < it.fend) {
        const int i = f / G, h = f - i * G;
        cp_async4(&sL[buf][threadIdx.x],
                  a.lse + (static_cast<int64_t>(layer) * a.hq + kvh * G + h) * a.total_tokens + t0 + i);
      }
    }
  };
  float colsum[kImpSlices][2];
#pragma unroll
  for (int u = 0; u < kImpSlices; ++u) colsum[u][0] = colsum[u][1] = 0.f;
  // a ring of kImpStages tiles: tile j lives in buffer j % kImpStages; one
  // barrier per tile both publishes tile j and retires tile j - 1's buffer
  ColTile tiles[kImpStages];  // tiles[j % kImpStages]: the tile staged there
  bool valid[kImpStages];
  ColTile it;
  bool more = seek(0, it);
#pragma unroll
  for (int j = 0; j < kImpStages - 1; ++j) {
    valid[j] = more;
    if (more) {
      tiles[j] = it;
      stage(it, j);
      more = advance(it);
    }
    cp_async_commit();
  }
  valid[kImpStages - 1] = false;
  for (int j = 0; valid[j % kImpStages]; ++j) {
    const int buf = j % kImpStages;
    cp_async_wait<kImpStages - 2>();  // tile j has landed (this thread's copies)
    __syncthreads();                  // ... everyone's; tile j - 1's buffer is free
    {
      const int nb = (j + kImpStages - 1) % kImpStages;
      valid[nb] = more;
      if (more) {
        tiles[nb] = it;
        stage(it, nb);
        more = advance(it);
      }
      cp_async_commit();
    }
    const ColTile cur = tiles[buf];
    const uint32_t sq = shared_addr(&sQ[buf][0]);
    // a full tile whose every row sees every key of the CTA: no mask
    const bool open = keys_full && cur.f0 + kImpCols <= cur.fend && cur.f0 / G >= pos_hi &&
                      (!local || (cur.f0 + kImpCols - 1) / G - pos_lo < W);
#pragma unroll 1
    for (int ng = 0; ng < kImpCols / 32; ++ng) {
      // four 8-column tiles at a time: 2 slices x 4 tiles = 8 independent
      // accumulator chains per warp.  Q^T as the B operand: ldmatrix
      // matrices (columns of tile nt, chunks 4 jj .. 4 jj + 3)
      uint32_t b[4][KS][2];
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
        for (int jj = 0; jj < KS / 2; ++jj) {
          const int line = (ng * 4 + q4) * 8 + (lane & 7), c = 4 * jj + (lane >> 3);
          uint32_t rr[4];
          ldsm_x4(sq + (line * CHUNKS + (c ^ (line & 7))) * 16, rr);
          b[q4][2 * jj][0] = rr[0];
          b[q4][2 * jj][1] = rr[1];
          b[q4][2 * jj + 1][0] = rr[2];
          b[q4][2 * jj + 1][1] = rr[3];
        }
      float c[kImpSlices][4][4];
#pragma unroll
      for (int u = 0; u < kImpSlices; ++u)
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) c[u][q4][0] = c[u][q4][1] = c[u][q4][2] = c[u][q4][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks)
#pragma unroll
        for (int u = 0; u < kImpSlices; ++u)
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) mma_16816(c[u][q4], ka[u][ks], b[q4][ks][0], b[q4][ks][1]);
      // c[u][q4][kk * 2 + cc]: key gq + 8 kk of slice u, column 2 tq + cc of tile q4
      if (open) {
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const float l2 = sL[buf][(ng * 4 + q4) * 8 + 2 * tq + cc] * kLog2e;
#pragma unroll
            for (int u = 0; u < kImpSlices; ++u)
#pragma unroll
              for (int kk = 0; kk < 2; ++kk)
                colsum[u][kk] += ex2_fast(fmaf(c[u][q4][kk * 2 + cc], a.scale_log2, -l2));
          }
        continue;
      }
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        int ci[2];
        bool cv[2];
        float l2[2];
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int col = (ng * 4 + q4) * 8 + 2 * tq + cc;
          const int f = cur.f0 + col;
          cv[cc] = f < cur.fend;
          ci[cc] = f / G;
          l2[cc] = sL[buf][col] * kLog2e;
        }
#pragma unroll
        for (int u = 0; u < kImpSlices; ++u)
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            const int pk = kpos[u][kk];
#pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int i = ci[cc];
              const bool vis = cv[cc] && pk <= i && (!local || i - pk < W);
              colsum[u][kk] += vis ? ex2_fast(fmaf(c[u][q4][kk * 2 + cc], a.scale_log2, -l2[cc]))
                                   : 0.f;
            }
          }
      }
    }
  }
  cp_async_wait<0>();
  // sum over the four lanes of each key and write this chunk's partial
  float* part = a.part + ((static_cast<int64_t>(layer) * a.hkv + kvh) * a.n_chunks + chunk) *
                             a.total_tokens + t0;
#pragma unroll
  for (int u = 0; u < kImpSlices; ++u)
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      float v = colsum[u][kk];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      if (tq == 0 && kpos[u][kk] != INT_MAX) part[kpos[u][kk]] = v;
    }
}

// 2. importance: the partials added over kv heads and chunks, in that order
__global__ void __launch_bounds__(256) importance_reduce_kernel(const __grid_constant__ ImpArgs a) {
  const int pos = blockIdx.x * blockDim.x + threadIdx.x, layer = blockIdx.y;
  if (pos >= a.total_tokens) return;
  float v = 0.f;
  for (int kvh = 0; kvh < a.hkv; ++kvh)
    for (int c = 0; c < a.n_chunks; ++c)
      v += a.part[((static_cast<int64_t>(layer) * a.hkv + kvh) * a.n_chunks + c) * a.total_tokens + pos];
  a.importance[static_cast<int64_t>(layer) * a.total_tokens + pos] = v;
}

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

// 3. the top-k tokens of one (request, layer)
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

template <int D, int G>
cudaError_t launch_importance_typed(const ImpArgs& a, int n_tables, int max_blocks,
                                    cudaStream_t stream) {
  constexpr size_t smem = static_cast<size_t>(kImpStages) * kImpCols * (D * 2 + 4);
  auto colsum = importance_colsum_kernel<D, G>;
  cudaError_t e = cudaFuncSetAttribute(colsum, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  colsum<<<dim3(n_tables, max_blocks, a.n_chunks), kImpThreads, smem, stream>>>(a);
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
  a.lse = in.lse;
  a.part = in.part;
  a.importance = in.importance;
  a.tokens = in.tokens;
  a.token_count = in.token_count;
  a.n_pages = in.n_pages;
  a.n_req = in.n_req;
  a.n_layers = in.n_layers;
  a.hq = in.hq;
  a.hkv = in.hkv;
  a.p = in.p;
  a.total_tokens = in.total_tokens;
  a.window = in.window;
  a.top_k = in.top_k;
  a.n_chunks = in.n_chunks;
  a.scale_log2 = in.softmax_scale * kLog2e;
  for (int k = 0; k < in.n_layers * in.hkv; ++k) a.cls[k] = in.cls[k];
  a.error_word = in.error_word;
  const int n_tables = in.n_req * in.n_layers * in.hkv;
  if (n_tables == 0) return cudaSuccess;
  const int G = in.hq / in.hkv;
  const int nb = in.max_blocks > 0 ? in.max_blocks : 1;
#define RK_IMP_CASE(DD, GG) \
  if (in.d == DD && G == GG) return launch_importance_typed<DD, GG>(a, n_tables, nb, stream);
  RK_IMP_CASE(128, 1) RK_IMP_CASE(128, 2) RK_IMP_CASE(128, 3) RK_IMP_CASE(128, 4)
  RK_IMP_CASE(128, 5) RK_IMP_CASE(128, 6) RK_IMP_CASE(128, 7) RK_IMP_CASE(128, 8)
  RK_IMP_CASE(64, 1) RK_IMP_CASE(64, 2) RK_IMP_CASE(64, 3) RK_IMP_CASE(64, 4)
  RK_IMP_CASE(64, 5) RK_IMP_CASE(64, 6) RK_IMP_CASE(64, 7) RK_IMP_CASE(64, 8)
#undef RK_IMP_CASE
  return cudaErrorInvalidValue;
}

}  // namespace rk
