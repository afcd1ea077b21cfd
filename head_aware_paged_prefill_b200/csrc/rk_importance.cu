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
//   1. column sums on the tensor cores, one 256-thread CTA per (table, 128
//      keys, row chunk).  The 128 keys of relocated K are the rows of the
//      A operand (staged once); tiles of 64 (row, q head) columns of Q are
//      the B operand, streamed with their lse through a four-deep cp.async
//      ring, only the rows of the table's row set that can see the keys
//      (causal from the lowest key, up to the highest key + W - 1 for local
//      tables).  S = K Q^T lands in TMEM, one lane per key; the weights
//      2^(S scale log2 e - lse log2 e), masked per element where a tile
//      straddles a causal or window edge, are summed by the thread that
//      owns the key's lane (two warps per lane quarter, 32 columns each).
//      A chunk is 8192 / G rows aligned on row 0, so the CTAs of a chunk
//      read the same Q rows from L2 and no CTA walks a whole long request;
//      each (layer, kv head, chunk, token) partial is written by exactly one
//      CTA.
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
#include "sm100.cuh"

namespace rk {

namespace {

constexpr int kImpSelectThreads = 1024;
constexpr float kLog2e = 1.4426950408889634f;

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

// 2^x on the special function unit (flushes results below 2^-126 to 0,
// which a sum of weights in [0, 1] does not notice)
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// A run of Q tile columns: flat (row, q head) indices [f0, fend), f = row G + h.
struct ColTile {
  int ri, f0, fend;
};

// 1. column sums of one table's 128 keys on the 5th-generation tensor cores:
// the keys are the 128 rows of A (one TMEM lane each), a Q tile of 64
// (row, q head) columns is B, and S = K Q^T lands in TMEM as 128 lanes x 64
// fp32 columns (two buffers).  Thread i owns key i: it reads its lane's 64
// scores and adds their weights without any cross-lane step.  The MMA of
// tile j + 1 is issued before the weights of tile j are taken, so the
// tensor work hides under the exponentials.  Operands are staged by
// cp.async straight into the 128-byte-swizzled K-major layout (16-byte
// chunk c of row r at c ^ (r & 7) inside 1024-byte atoms).
constexpr int kTcCols = 64;     // Q tile columns (MMA N)
constexpr int kTcQBufs = 4;     // Q / lse tiles in flight
constexpr int kTcTmemCols = 128;  // two S buffers of kTcCols fp32 columns
constexpr int kTcThreads = 256;   // two warps per TMEM lane quarter, each half the columns

template <int D>
struct TcSmem {
  static constexpr int kKBytes = 128 * D * 2;
  static constexpr int kQBytes = kTcCols * D * 2;
  static constexpr int kOffQ = kKBytes;
  static constexpr int kOffL = kOffQ + kTcQBufs * kQBytes;
  static constexpr int kOffBar = kOffL + kTcQBufs * kTcCols * 4;
  static constexpr int kBytes = kOffBar + 64;
  static constexpr int kAlloc = kBytes + 1024;  // room to align the base to 1024
};

template <int D, int G>
__global__ void __launch_bounds__(kTcThreads)
    importance_colsum_tc_kernel(const __grid_constant__ ImpArgs a) {
  using S = TcSmem<D>;
  constexpr int CHUNKS = D / 8;
  extern __shared__ uint8_t tc_raw[];
  uint8_t* sm = tc_raw + ((1024 - (smem_u32(tc_raw) & 1023)) & 1023);
  uint8_t* sK = sm;
  uint8_t* sQ = sm + S::kOffQ;
  float* sL = reinterpret_cast<float*>(sm + S::kOffL);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + S::kOffBar);  // [2] S full
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + S::kOffBar + 16);
  int* abort_flag = reinterpret_cast<int*>(sm + S::kOffBar + 20);
  const int warp = threadIdx.x >> 5, tid = threadIdx.x;
  const int key = tid & 127;      // TMEM lane = row of the K tile
  const int half = warp >> 2;     // which 32 of the tile's 64 columns
  const int t = blockIdx.x;
  const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
  const int n_e = a.entry_count[t], e_first = a.entry_start[t], rc = a.range_count[t];
  const int spp = a.p / 16;
  const int n_sl = n_e * spp;
  const int s_begin = blockIdx.y * 8;
  if (s_begin >= n_sl || rc == 0) return;
  const int s_end = min(n_sl, s_begin + 8);
  const int t0 = a.cu[r], L = a.cu[r + 1] - t0;
  const bool local = a.cls[layer * a.hkv + kvh] == RK_LOCAL;
  const int W = a.window;
  int pos_lo, pos_hi;
  {
    const rk_entry e0 = a.entries[e_first + s_begin / spp];
    pos_lo = e0.logical_pos + (s_begin % spp) * 16;
    const int sl = s_end - 1;
    const rk_entry e1 = a.entries[e_first + sl / spp];
    pos_hi = e1.logical_pos + min((sl % spp) * 16 + 16, e1.n_valid) - 1;
  }
  constexpr int RPC = kImpChunkCols / G;
  const int chunk = blockIdx.z;
  const int row_lo = max(pos_lo, chunk * RPC);
  const int row_hi =
      min(local ? min(L - 1, pos_hi + min(W, L) - 1) : L - 1, chunk * RPC + RPC - 1);
  if (row_lo > row_hi) return;
  // this thread's key (TMEM lane `key` = row `key` of the K tile)
  int kpos = INT_MAX;
  {
    const int s = s_begin + key / 16, kk = key % 16;
    if (s < s_end) {
      const rk_entry en = a.entries[e_first + s / spp];
      const int k0 = (s % spp) * 16;
      if (en.phys_page >= 0 && en.phys_page < a.n_pages && k0 + kk < en.n_valid)
        kpos = en.logical_pos + k0 + kk;
    }
  }
  // stage the K tile: row rr <- key rr of the CTA (zeros for no key)
  for (int x = tid; x < 128 * CHUNKS; x += kTcThreads) {
    const int rr = x / CHUNKS, c = x % CHUNKS;
    uint8_t* dst = sK + (c >> 3) * (128 * 128) + rr * 128 + (((c & 7) ^ (rr & 7)) << 4);
    const int s = s_begin + rr / 16;
    bool copied = false;
    if (s < s_end) {
      const rk_entry en = a.entries[e_first + s / spp];
      if (en.phys_page >= 0 && en.phys_page < a.n_pages) {
        const int64_t row = static_cast<int64_t>(en.phys_page) * a.p + (s % spp) * 16 + rr % 16;
        cp_async16(dst, a.k_pool + row * D + c * 8);
        copied = true;
      } else if (rr % 16 == 0 && c == 0) {
        atomicOr(a.error_word, static_cast<int>(RK_DEV_BAD_PAGE));
      }
    }
    if (!copied) *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
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
    it.f0 += kTcCols;
    if (it.f0 < it.fend) return true;
    return seek(it.ri + 1, it);
  };
  // stage a Q tile (its columns' rows, zeros past the run) and its lse
  auto stage = [&](const ColTile& it, int buf) {
    uint8_t* q = sQ + buf * S::kQBytes;
    for (int x = tid; x < kTcCols * CHUNKS; x += kTcThreads) {
      const int n = x / CHUNKS, c = x % CHUNKS;
      uint8_t* dst = q + (c >> 3) * (kTcCols * 128) + n * 128 + (((c & 7) ^ (n & 7)) << 4);
      const int f = it.f0 + n;
      if (f < it.fend) {
        const int i = f / G, h = f - i * G;
        cp_async16(dst, a.q + ((static_cast<int64_t>(layer) * a.total_tokens + t0 + i) * a.hq +
                               kvh * G + h) * D + c * 8);
      } else {
        *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    if (tid < kTcCols) {
      const int f = it.f0 + tid;
      if (f < it.fend) {
        const int i = f / G, h = f - i * G;
        cp_async4(&sL[buf * kTcCols + tid],
                  a.lse + (static_cast<int64_t>(layer) * a.hq + kvh * G + h) * a.total_tokens + t0 + i);
      }
    }
  };
  ColTile tiles[kTcQBufs];
  int n_staged = 0;
  ColTile it;
  bool more = seek(0, it);
  auto stage_next = [&]() {
    if (more) {
      tiles[n_staged % kTcQBufs] = it;
      stage(it, n_staged % kTcQBufs);
      ++n_staged;
      more = advance(it);
    }
    cp_async_commit();  // one group per call, empty or not
  };
  stage_next();  // group 0: the K tile and Q tile 0
  stage_next();  // Q tile 1
  stage_next();  // Q tile 2
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, kTcTmemCols);
    tmem_relinquish();
  }
  const bool keys_full = __syncthreads_and(kpos != INT_MAX);
  const WaitCtx wc{abort_flag, a.error_word, a.error_word + 1};
  cp_async_wait<2>();  // K and Q tile 0 have landed (this thread's copies)
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  constexpr uint32_t idesc = idesc_bf16_f32(128, kTcCols, false);
  const uint32_t sK_u = smem_u32(sK), sQ_u = smem_u32(sQ);
  auto issue = [&](int j) {  // S buffer j & 1 <- K Q_j^T
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t ad = desc_sw128(sK_u + (kk >> 2) * (128 * 128) + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = desc_sw128(
          sQ_u + (j % kTcQBufs) * S::kQBytes + (kk >> 2) * (kTcCols * 128) + (kk & 3) * 32, 16, 1024);
      mma_bf16_ss(tmem + (j & 1) * kTcCols, ad, bd, idesc, kk > 0 ? 1u : 0u);
    }
    tc_commit(&bars[j & 1]);
  };
  int n_issued = 0, n_waited = 0;
  if (tid == 0 && n_staged > 0) issue(0);
  if (n_staged > 0) n_issued = 1;
  float acc0 = 0.f, acc1 = 0.f;
  bool ok = true;
  const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
  for (int j = 0; j < n_staged; ++j) {
    cp_async_wait<1>();  // tile j + 1 has landed (this thread's copies)
    fence_proxy_async_smem();
    tc_fence_before();
    ok = __syncthreads_and(ok);  // ... everyone's; tile j - 1 is fully consumed
    if (!ok) break;
    tc_fence_after();
    stage_next();  // tile j + 3 into tile j - 1's buffer
    if (j + 1 < n_staged) {
      if (tid == 0) issue(j + 1);
      ++n_issued;
    }
    ok = mbar_wait(&bars[j & 1], (j >> 1) & 1, wc, 1);
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) continue;  // the next barrier ends the loop for everyone
    ++n_waited;
    tc_fence_after();
    const ColTile cur = tiles[j % kTcQBufs];
    const float* lse = sL + (j % kTcQBufs) * kTcCols;
    const bool open = keys_full && cur.f0 + kTcCols <= cur.fend && cur.f0 / G >= pos_hi &&
                      (!local || (cur.f0 + kTcCols - 1) / G - pos_lo < W);
    {
      const int c0 = half * 32;
      uint32_t v[32];
      tmem_ld_x32(tmem + lane_base + (j & 1) * kTcCols + c0, v);
      tmem_ld_wait(v);
      if (open) {
#pragma unroll
        for (int n = 0; n < 32; n += 2) {
          acc0 += ex2_fast(fmaf(__uint_as_float(v[n]), a.scale_log2, -lse[c0 + n] * kLog2e));
          acc1 += ex2_fast(fmaf(__uint_as_float(v[n + 1]), a.scale_log2, -lse[c0 + n + 1] * kLog2e));
        }
      } else {
#pragma unroll
        for (int n = 0; n < 32; ++n) {
          const int f = cur.f0 + c0 + n;
          const int i = f / G;
          const bool vis = f < cur.fend && kpos <= i && (!local || i - kpos < W);
          const float w =
              vis ? ex2_fast(fmaf(__uint_as_float(v[n]), a.scale_log2, -lse[c0 + n] * kLog2e)) : 0.f;
          if (n & 1)
            acc1 += w;
          else
            acc0 += w;
        }
      }
    }
    tc_fence_before();
  }
  cp_async_wait<0>();
  if (tid == 0) {
    // MMAs still in flight after an abort (at most two, one per barrier):
    // let them finish before the TMEM goes
    for (int m = n_waited; m < n_issued; ++m) mbar_wait_drain(&bars[m & 1], (m >> 1) & 1);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
  // the two column halves of each key, added in a fixed order
  float* red = reinterpret_cast<float*>(sm + S::kOffL);
  if (half == 1) red[key] = acc0 + acc1;
  __syncthreads();
  if (half == 0 && ok && kpos != INT_MAX)
    a.part[((static_cast<int64_t>(layer) * a.hkv + kvh) * a.n_chunks + chunk) * a.total_tokens +
           t0 + kpos] = (acc0 + acc1) + red[key];
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
  constexpr size_t smem = TcSmem<D>::kAlloc;
  auto colsum = importance_colsum_tc_kernel<D, G>;
  cudaError_t e = cudaFuncSetAttribute(colsum, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  colsum<<<dim3(n_tables, max_blocks, a.n_chunks), kTcThreads, smem, stream>>>(a);
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
