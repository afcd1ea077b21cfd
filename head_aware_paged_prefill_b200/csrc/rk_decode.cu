// SegPaged decode: one query row per (request, layer, q head), the last
// position of each request, over the per-head page tables rk_select_visible
// built (RedKnot pages: the SegPagedAttention runtime serves the per-head
// visible windows; paooo page, "application scenarios": in streaming
// generation the local heads keep reading their recent paged KV).  A decode
// step appends a token to each request's uncached tail; its row attends to
// the table's visible keys under the class rule, as the prefill's last row
// does.
//
// HBM bound: every visible key and value is read once per kv head, for all
// G q heads of the group.  Split-K flash decode with balanced splits:
//   1. the tables' decode pages, concatenated in table order, are cut on the
//      host into equal ranges, one per CTA (two CTAs per SM, one wave), so
//      every CTA streams the same number of pages.  A CTA walks its range
//      table by table; each piece (the range's part in one table) is
//      streamed by the CTA's warps, each through a private cp.async ring of
//      16-key slices, running Q K^T and P V of the GQA group as warp-level
//      bf16 MMAs (the G heads are the rows of a 16-row tile) with its own
//      online softmax; the warps merge at the piece's end and the piece
//      writes (o, m, l);
//   2. one CTA per table merges its pieces in order: o = sum_s o_s
//      2^(m_s - M) / L, lse = (M + log2 L) ln 2, written as bf16 / fp32.
// The MMAs are there to cut instruction issue (the CUDA-core form of the
// same dot products issued ~5x more instructions per byte and reached a
// third of the HBM bandwidth); the bound stays the HBM stream.  Warp-level
// MMAs rather than tcgen05: a 16-row tile already wastes 16 / G of the
// rows, tcgen05's smallest tile has 64, and per-warp tiles keep the warps
// independent.
// Relocated pools are read (the cached pages' RoPE delta is applied by
// rk_relocate_rope beforehand), so the entry's delta is not used here.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "rk_internal.h"

namespace rk {

namespace {

constexpr int kDecodeThreads = 128;
constexpr int kDecodeStages = 3;  // ring depth of each warp

struct DecodeArgs {
  const __nv_bfloat16* q;  // [n_layers][n_req][hq][d]
  const __nv_bfloat16* k_pool;
  const __nv_bfloat16* v_pool;
  const rk_entry* entries;
  const int32_t* entry_start;
  const int32_t* entry_count;
  const rk_range* ranges;
  const int32_t* range_start;
  const int32_t* range_count;
  const int32_t* req_len;  // [n_req]
  const DecodeTable* tables;  // [n_tables]
  __nv_bfloat16* o;  // [n_layers][n_req][hq][d]
  float* lse;        // [n_layers][hq][n_req] or null
  float* part_o;     // [pieces][g][d]
  float* part_ml;    // [pieces][g][2]
  int64_t n_pages;
  int n_req, n_layers, hq, hkv, g, p, n_cta, per, total, window;
  float scale_log2;  // softmax scale * log2(e)
  int8_t cls[kDecodeMaxLh];
  int32_t* error_word;
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t shared_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// Four 8x8 bf16 matrices from shared memory; lanes 8i..8i+7 address the
// rows of matrix i, and lane l receives row l / 4, columns 2 (l % 4) + {0, 1}
// of each (.trans: row and column swapped).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}

// c (16 x 8, fp32) += A (16 x 16, bf16) B (16 x 8, bf16).  A's rows 8..15 are
// zero here (they would be q heads G + 8 and up), so only its fragments for
// rows 0..7 are passed.
__device__ __forceinline__ void mma_rows8(float (&c)[4], uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// 1. one piece: entries [e0, e0 + n_ent) of table t's page table, result
// into partial `part`.  The piece's pages are cut into 16-key slices
// (P / 16 per page); warp w takes slices w, w + NW, ... and streams them
// through its own ring of kDecodeStages shared-memory buffers by cp.async,
// so the warps never wait for one another inside the loop.  Per slice:
//   S (G x 16) = Q K^T and O += P V as m16n8k16 bf16 MMAs with fp32
//   accumulators, the G q heads of the kv head as the rows (padded to 16);
//   an online softmax per head in the warp (row max over the 4 lanes that
//   hold a row).
// Rows of K and V are stored with their 16-byte chunks permuted (chunk c of
// key k at c ^ (k & 7)), so that the eight rows each ldmatrix reads fall in
// distinct banks.  At the end the warps' (m, l, o) are merged in shared
// memory and the piece writes (o, m, l).
template <int D, int G>
__device__ void decode_piece(const DecodeArgs& a, int t, int e0, int n_ent, int64_t part,
                             uint8_t* smem) {
  constexpr int NW = kDecodeThreads / 32;
  constexpr int KS = D / 16;      // 16-column steps of Q K^T; pairs of 8-column tiles of P V
  constexpr int CHUNKS = D / 8;   // 16-byte chunks of a key row
  constexpr int SLICE = 16 * D;   // elements of one slice of K (or V)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, tq = lane & 3;  // fragment row (q head) and column pair
  const int P = a.p;
  const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
  const int e_first = a.entry_start[t];
  const int row = a.req_len[r] - 1;  // the request's last position
  const int cls = a.cls[layer * a.hkv + kvh];
  const int lo = cls == RK_LOCAL ? row - a.window + 1 : 0;  // first visible key
  __syncthreads();  // the previous piece's merge is done with the shared memory
  const int spp = P / 16;
  const int n_slices = n_ent * spp;
  const int my_n = warp < n_slices ? (n_slices - warp + NW - 1) / NW : 0;
  __nv_bfloat16* ring =
      reinterpret_cast<__nv_bfloat16*>(smem) + warp * (kDecodeStages * 2 * SLICE);
  // Q as the A operand, rows = q heads: columns 16 ks + 2 tq (+8) of head gq
  uint32_t qa[KS][2];
  {
    const bool real = gq < G;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(
        a.q + ((static_cast<int64_t>(layer) * a.n_req + r) * a.hq + kvh * G + (real ? gq : 0)) * D);
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qa[ks][0] = real ? q32[ks * 8 + tq] : 0u;
      qa[ks][1] = real ? q32[ks * 8 + 4 + tq] : 0u;
    }
  }
  // stage this warp's i-th slice into ring buffer i % kDecodeStages (a page
  // outside the pool is not copied and is skipped below, flagged once)
  auto stage = [&](int i) {
    const int sg = warp + NW * i;
    const rk_entry en = a.entries[e_first + e0 + sg / spp];
    if (en.phys_page < 0 || en.phys_page >= a.n_pages) return;
    const int64_t base = (static_cast<int64_t>(en.phys_page) * P + (sg % spp) * 16) * D;
    const uint4* gk = reinterpret_cast<const uint4*>(a.k_pool + base);
    const uint4* gv = reinterpret_cast<const uint4*>(a.v_pool + base);
    uint4* sk = reinterpret_cast<uint4*>(ring + (i % kDecodeStages) * 2 * SLICE);
    uint4* sv = sk + SLICE / 8;
#pragma unroll
    for (int u = 0; u < 16 * CHUNKS / 32; ++u) {
      const int x = lane + 32 * u, key = x / CHUNKS, c = x % CHUNKS;
      const int dst = key * CHUNKS + (c ^ (key & 7));
      cp_async16(sk + dst, gk + x);
      cp_async16(sv + dst, gv + x);
    }
  };
#pragma unroll
  for (int i = 0; i < kDecodeStages - 1; ++i) {
    if (i < my_n) stage(i);
    cp_async_commit();
  }
  float acc[2 * KS][4];
#pragma unroll
  for (int n = 0; n < 2 * KS; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  float m_run = -INFINITY;  // row gq's running max (log2 domain)
  float l_run = 0.f;        // this lane's share of row gq's running sum
  // ldmatrix row addresses: for K, matrices (keys 0-7 | 8-15) x (chunk 2ks | 2ks+1);
  // for V (transposed), (keys 0-7 | 8-15) x (chunk 2np | 2np+1)
  const int k_key = ((lane >> 4) << 3) | (lane & 7), k_c = (lane >> 3) & 1;
  const int v_key = (((lane >> 3) & 1) << 3) | (lane & 7), v_c = lane >> 4;
  for (int i = 0; i < my_n; ++i) {
    if (i + kDecodeStages - 1 < my_n) stage(i + kDecodeStages - 1);
    cp_async_commit();
    cp_async_wait<kDecodeStages - 1>();  // slice i has landed (this lane's copies)
    __syncwarp();                        // ... and every lane's
    const int sg = warp + NW * i;
    const rk_entry en = a.entries[e_first + e0 + sg / spp];
    if (en.phys_page < 0 || en.phys_page >= a.n_pages) {
      if (lane == 0) atomicOr(a.error_word, static_cast<int>(RK_DEV_BAD_PAGE));
      continue;  // nothing was read from this buffer
    }
    const int k0 = (sg % spp) * 16;
    const uint32_t sk = shared_addr(ring + (i % kDecodeStages) * 2 * SLICE);
    const uint32_t sv = sk + SLICE * 2;
    float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      uint32_t b[4];
      const int c = 2 * ks + k_c;
      ldsm_x4(sk + (k_key * CHUNKS + (c ^ (k_key & 7))) * 16, b);
      mma_rows8(s[0], qa[ks][0], qa[ks][1], b[0], b[1]);
      mma_rows8(s[1], qa[ks][0], qa[ks][1], b[2], b[3]);
    }
    // lane holds S[gq][8 nt + 2 tq + cc]
    float sc[2][2];
    float mx = -INFINITY;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int j = k0 + nt * 8 + 2 * tq + cc;  // key within the page
        const int pos = en.logical_pos + j;
        const bool vis = j < en.n_valid && pos <= row && pos >= lo;
        sc[nt][cc] = vis ? s[nt][cc] * a.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sc[nt][cc]);
      }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m_run, mx);
    const float m_use = m_new == -INFINITY ? 0.f : m_new;
    const float alpha = exp2f(m_run - m_use);
    float p[2][2];
    float psum = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        p[nt][cc] = exp2f(sc[nt][cc] - m_use);
        psum += p[nt][cc];
      }
    l_run = l_run * alpha + psum;
    m_run = m_new;
    // P as the A operand: row gq, keys 2 tq (+8) of the slice
    const uint32_t pa0 = pack_bf16x2(p[0][0], p[0][1]);
    const uint32_t pa2 = pack_bf16x2(p[1][0], p[1][1]);
#pragma unroll
    for (int n = 0; n < 2 * KS; ++n) {
      acc[n][0] *= alpha;
      acc[n][1] *= alpha;
    }
#pragma unroll
    for (int np = 0; np < KS; ++np) {
      uint32_t b[4];
      const int c = 2 * np + v_c;
      ldsm_x4_trans(sv + (v_key * CHUNKS + (c ^ (v_key & 7))) * 16, b);
      mma_rows8(acc[2 * np], pa0, pa2, b[0], b[1]);
      mma_rows8(acc[2 * np + 1], pa0, pa2, b[2], b[3]);
    }
    __syncwarp();  // the buffer is restaged next iteration
  }
  cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();  // every warp is done with its ring: reuse it for the merge
  float* sO = reinterpret_cast<float*>(smem);  // [NW][G][D]
  float* sML = sO + NW * G * D;                // [NW][G][2]
  if (gq < G) {
#pragma unroll
    for (int n = 0; n < 2 * KS; ++n) {
      sO[(warp * G + gq) * D + n * 8 + 2 * tq] = acc[n][0];
      sO[(warp * G + gq) * D + n * 8 + 2 * tq + 1] = acc[n][1];
    }
    if (tq == 0) {
      sML[(warp * G + gq) * 2] = m_run;
      sML[(warp * G + gq) * 2 + 1] = l_run;
    }
  }
  __syncthreads();
  for (int x = threadIdx.x; x < G * D; x += kDecodeThreads) {
    const int h = x / D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, sML[(w * G + h) * 2]);
    float tot = 0.f, L = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float m = sML[(w * G + h) * 2];
        if (m == -INFINITY) continue;
        const float f = exp2f(m - M);
        tot += sO[w * G * D + x] * f;
        L += sML[(w * G + h) * 2 + 1] * f;
      }
    }
    a.part_o[part * G * D + x] = tot;
    if (x % D == 0) {
      a.part_ml[(part * G + h) * 2] = M;
      a.part_ml[(part * G + h) * 2 + 1] = L;
    }
  }
}

// 1'. the CTA's range [c per, (c + 1) per) of the concatenated decode pages,
// piece by piece (the range's part in each table it crosses)
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int c = blockIdx.x, n_tables = a.n_req * a.n_layers * a.hkv;
  int a0 = c * a.per;
  const int a1 = min(a.total, a0 + a.per);
  int lo = 0, hi = n_tables;  // last table with g0 <= a0
  while (hi - lo > 1) {
    const int m = (lo + hi) >> 1;
    if (a.tables[m].g0 <= a0) lo = m; else hi = m;
  }
  int t = lo;
  while (a0 < a1) {
    while (t < n_tables && a.tables[t].g0 + a.tables[t].n_dec <= a0) ++t;
    if (t >= n_tables) break;
    const DecodeTable dt = a.tables[t];
    const int end = min(a1, dt.g0 + dt.n_dec);
    const int64_t part = static_cast<int64_t>(dt.piece_base) + (c - dt.c_first);
    if (a.entry_count[t] == dt.n_e) {
      decode_piece<D, G>(a, t, dt.first + (a0 - dt.g0), end - a0, part, smem);
    } else {  // page tables of another layout: an empty partial, flagged
      if (threadIdx.x == 0) atomicOr(a.error_word, static_cast<int>(RK_DEV_CAPACITY));
      for (int x = threadIdx.x; x < G * D; x += kDecodeThreads) a.part_o[part * G * D + x] = 0.f;
      for (int x = threadIdx.x; x < G; x += kDecodeThreads) {
        a.part_ml[(part * G + x) * 2] = -INFINITY;
        a.part_ml[(part * G + x) * 2 + 1] = 0.f;
      }
    }
    a0 = end;
  }
}

// 2. merge the pieces of one table, in order
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
  const int t = blockIdx.x;
  const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
  const DecodeTable dt = a.tables[t];
  if (dt.n_dec == 0) return;  // the request's last position is not a row of this table
  const int64_t base = dt.piece_base;
  for (int x = threadIdx.x; x < G * D; x += kDecodeThreads) {
    const int h = x / D, c = x % D;
    float M = -INFINITY;
    for (int s = 0; s < dt.n_pieces; ++s) M = fmaxf(M, a.part_ml[((base + s) * G + h) * 2]);
    float L = 0.f, acc = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < dt.n_pieces; ++s) {
        const float m = a.part_ml[((base + s) * G + h) * 2];
        if (m == -INFINITY) continue;
        const float f = exp2f(m - M);
        L += a.part_ml[((base + s) * G + h) * 2 + 1] * f;
        acc += a.part_o[((base + s) * G + h) * D + c] * f;
      }
    }
    const int qh = kvh * G + h;
    const int64_t oi = ((static_cast<int64_t>(layer) * a.n_req + r) * a.hq + qh) * D + c;
    a.o[oi] = __float2bfloat16_rn(L > 0.f ? acc / L : 0.f);
    if (a.lse && c == 0) {
      const int64_t li = (static_cast<int64_t>(layer) * a.hq + qh) * a.n_req + r;
      a.lse[li] = L > 0.f ? (M + log2f(L)) * 0.69314718055994531f : -INFINITY;
    }
  }
}

template <int D, int G>
cudaError_t launch_decode_typed(const DecodeArgs& a, int n_tables, cudaStream_t stream) {
  constexpr int NW = kDecodeThreads / 32;
  constexpr size_t ring = static_cast<size_t>(NW) * kDecodeStages * 2 * 16 * D * sizeof(__nv_bfloat16);
  constexpr size_t merge = static_cast<size_t>(NW) * G * (D + 2) * sizeof(float);
  const size_t smem = ring > merge ? ring : merge;
  auto split = decode_split_kernel<D, G>;
  cudaError_t e = cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  split<<<a.n_cta, kDecodeThreads, smem, stream>>>(a);
  decode_combine_kernel<D, G><<<n_tables, kDecodeThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunchArgs& in, cudaStream_t stream) {
  DecodeArgs a{};
  a.q = static_cast<const __nv_bfloat16*>(in.q);
  a.k_pool = static_cast<const __nv_bfloat16*>(in.k_pool);
  a.v_pool = static_cast<const __nv_bfloat16*>(in.v_pool);
  a.entries = in.entries;
  a.entry_start = in.entry_start;
  a.entry_count = in.entry_count;
  a.ranges = in.ranges;
  a.range_start = in.range_start;
  a.range_count = in.range_count;
  a.req_len = in.req_len;
  a.tables = in.tables;
  a.o = static_cast<__nv_bfloat16*>(in.o);
  a.lse = in.lse;
  a.part_o = in.part_o;
  a.part_ml = in.part_ml;
  a.n_pages = in.n_pages;
  a.n_req = in.n_req;
  a.n_layers = in.n_layers;
  a.hq = in.hq;
  a.hkv = in.hkv;
  a.g = in.hq / in.hkv;
  a.p = in.p;
  a.n_cta = in.n_cta;
  a.per = in.per;
  a.total = in.total;
  a.window = in.window;
  a.scale_log2 = in.softmax_scale * 1.4426950408889634f;
  for (int k = 0; k < in.n_layers * in.hkv; ++k) a.cls[k] = in.cls[k];
  a.error_word = in.error_word;
  const int n_tables = in.n_req * in.n_layers * in.hkv;
  if (n_tables == 0 || in.total == 0) return cudaSuccess;
  const int G = a.g;
#define RK_DECODE_CASE(DD, GG) \
  if (in.d == DD && G == GG) return launch_decode_typed<DD, GG>(a, n_tables, stream);
  RK_DECODE_CASE(128, 1) RK_DECODE_CASE(128, 2) RK_DECODE_CASE(128, 3) RK_DECODE_CASE(128, 4)
  RK_DECODE_CASE(128, 5) RK_DECODE_CASE(128, 6) RK_DECODE_CASE(128, 7) RK_DECODE_CASE(128, 8)
  RK_DECODE_CASE(64, 1) RK_DECODE_CASE(64, 2) RK_DECODE_CASE(64, 3) RK_DECODE_CASE(64, 4)
  RK_DECODE_CASE(64, 5) RK_DECODE_CASE(64, 6) RK_DECODE_CASE(64, 7) RK_DECODE_CASE(64, 8)
#undef RK_DECODE_CASE
  return cudaErrorInvalidValue;
}

}  // namespace rk
