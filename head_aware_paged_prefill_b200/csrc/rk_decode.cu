// SegPaged decode: one query row per (request, layer, q head), the last
// position of each request, over the per-head page tables rk_select_visible
// built (RedKnot pages: the SegPagedAttention runtime serves the per-head
// visible windows; paooo page, "how to use": generation streams after the
// prefill).  A decode step appends a token to each request's uncached tail;
// its row attends to the table's visible keys under the class rule, as the
// prefill's last row does.
//
// HBM bound (every visible key and value is read once per q-head group), so
// the kernel is a split-K flash decode on the CUDA cores:
//   1. one CTA per (table, split of kDecodePages pages) for all G q heads of
//      the kv head: K and V pages are staged in shared memory by cp.async,
//      two buffers deep; each lane owns D / 32 columns (its slice of the G
//      queries in registers), each warp a quarter of a page's keys, and the
//      per-(key, head) partial dots are summed over the lanes 32 values per
//      transposing butterfly; an online softmax per head keeps (m, l), each
//      warp its share of the output; the split writes (o, m, l);
//   2. one CTA per table merges its splits: o = sum_s o_s e^(m_s - M) / L,
//      lse = M + ln L, written as bf16 / fp32.
// Relocated pools are read (the cached pages' RoPE delta is applied by
// rk_relocate_rope beforehand), so the entry's delta is not used here.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>

#include "rk_internal.h"

namespace rk {

namespace {

constexpr int kDecodeThreads = 128;

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
  __nv_bfloat16* o;  // [n_layers][n_req][hq][d]
  float* lse;        // [n_layers][hq][n_req] or null
  float* part_o;     // [n_tables][max_splits][g][d]
  float* part_ml;    // [n_tables][max_splits][g][2]
  int64_t n_pages;
  int n_req, n_layers, hq, hkv, g, p, max_splits, window;
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

// Sum over the 32 lanes of each of 32 values: after the call, lane l holds in
// v[0] the total of value index l (five exchange steps, 31 shuffles).
__device__ __forceinline__ void warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16, n = 32; off >= 1; off >>= 1, n >>= 1) {
    const bool upper = lane & off;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? v[i] : v[i + n / 2];
      const float keep = upper ? v[i + n / 2] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
}

// 1. one split of one table.  Lane l of every warp owns columns
// [l * CPL, (l + 1) * CPL) and holds those columns of the G queries; warp w
// takes keys [w * KPW, (w + 1) * KPW) of each page.  Pages are staged by
// cp.async, two buffers deep.
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int CPL = D / 32;
  constexpr int NW = kDecodeThreads / 32;
  extern __shared__ __align__(16) uint8_t smem[];
  const int P = a.p;
  const int KPW = P / NW;  // keys of a page per warp (16 at P 64, 4 at P 16)
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);  // [2][64][D]
  __nv_bfloat16* sV = sK + 2 * 64 * D;                        // [2][64][D]
  float* sP = reinterpret_cast<float*>(sV + 2 * 64 * D);       // [G][64] scores, then weights
  float* sM = sP + G * 64;                                    // [G] running max (log2 domain)
  float* sL = sM + G;                                         // [G] running sum
  float* sA = sL + G;                                         // [G] rescale of this page
  float* sO = sA + G;                                         // [NW][G][D] warp partials
  const int t = blockIdx.x, split = blockIdx.y;
  const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
  const int n_e = a.entry_count[t], e_first = a.entry_start[t];
  const int e0 = split * kDecodePages;
  const int64_t part = static_cast<int64_t>(t) * a.max_splits + split;
  const int row = a.req_len[r] - 1;  // the request's last position
  // the row must belong to the table's row set (else the combine skips it too)
  const int rc = a.range_count[t];
  if (n_e == 0 || rc == 0 || a.ranges[a.range_start[t] + rc - 1].end != row + 1) return;
  const int cls = a.cls[layer * a.hkv + kvh];
  const int lo = cls == RK_LOCAL ? row - a.window + 1 : 0;  // first visible key
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // this lane's columns of the G queries, scaled into the log2 domain
  float qr[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      const int64_t qi = ((static_cast<int64_t>(layer) * a.n_req + r) * a.hq + kvh * G + h) * D +
                         lane * CPL + k;
      qr[h][k] = __bfloat162float(a.q[qi]) * a.scale_log2;
    }
  float acc[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < CPL; ++k) acc[h][k] = 0.f;
  if (threadIdx.x < G) {
    sM[threadIdx.x] = -INFINITY;
    sL[threadIdx.x] = 0.f;
  }
  const int e_end = min(n_e, e0 + kDecodePages);
  // stage page e into buffer b (16-byte chunks; a page outside the pool is
  // not copied and is skipped below, flagged once)
  auto stage = [&](int e, int b) {
    const rk_entry en = a.entries[e_first + e];
    if (en.phys_page < 0 || en.phys_page >= a.n_pages) return;
    const uint4* gk = reinterpret_cast<const uint4*>(a.k_pool + static_cast<int64_t>(en.phys_page) * P * D);
    const uint4* gv = reinterpret_cast<const uint4*>(a.v_pool + static_cast<int64_t>(en.phys_page) * P * D);
    uint4* k4 = reinterpret_cast<uint4*>(sK + b * 64 * D);
    uint4* v4 = reinterpret_cast<uint4*>(sV + b * 64 * D);
    for (int x = threadIdx.x; x < P * D / 8; x += kDecodeThreads) {
      cp_async16(k4 + x, gk + x);
      cp_async16(v4 + x, gv + x);
    }
  };
  if (e0 < e_end) stage(e0, 0);
  cp_async_commit();
  for (int e = e0; e < e_end; ++e) {
    const int b = (e - e0) & 1;
    if (e + 1 < e_end) stage(e + 1, b ^ 1);
    cp_async_commit();
    cp_async_wait<1>();  // page e has landed
    __syncthreads();
    const rk_entry en = a.entries[e_first + e];
    if (en.phys_page < 0 || en.phys_page >= a.n_pages) {
      if (threadIdx.x == 0) atomicOr(a.error_word, static_cast<int>(RK_DEV_BAD_PAGE));
      __syncthreads();
      continue;  // uniform across the CTA
    }
    const __nv_bfloat16* kb = sK + b * 64 * D;
    const __nv_bfloat16* vb = sV + b * 64 * D;
    // scores of this warp's keys: partial dots over the lane's columns,
    // summed over the lanes 32 values at a time; a group holds KG whole keys
    // (value kk * G + h), the spare lanes zero
    constexpr int KG = 32 / G;
    const int j0 = warp * KPW;
    for (int kb0 = 0; kb0 < KPW; kb0 += KG) {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KG; ++kk) {
        if (kb0 + kk < KPW) {
          const __nv_bfloat16* kr = kb + (j0 + kb0 + kk) * D + lane * CPL;
          float kf[CPL];
          if constexpr (CPL == 4) {
            const uint2 raw = *reinterpret_cast<const uint2*>(kr);
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
            const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
            kf[0] = x.x; kf[1] = x.y; kf[2] = y.x; kf[3] = y.y;
          } else {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(kr));
            kf[0] = x.x; kf[1] = x.y;
          }
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float d0 = 0.f;
#pragma unroll
            for (int k = 0; k < CPL; ++k) d0 = fmaf(qr[h][k], kf[k], d0);
            v[kk * G + h] = d0;
          }
        }
      }
      warp_transpose_sum(v, lane);
      const int kk = lane / G, h = lane - kk * G;
      if (kk < KG && kb0 + kk < KPW) {
        const int j = j0 + kb0 + kk;
        const int pos = en.logical_pos + j;
        const bool vis = j < en.n_valid && pos <= row && pos >= lo;
        sP[h * 64 + j] = vis ? v[0] : -INFINITY;
      }
    }
    __syncthreads();
    // per head (one warp each): new running max, weights p = 2^(s - m),
    // rescale factor
    for (int h = warp; h < G; h += NW) {
      float mx = -INFINITY;
      for (int j = lane; j < P; j += 32) mx = fmaxf(mx, sP[h * 64 + j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = sM[h];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int j = lane; j < P; j += 32) {
        const float sc = sP[h * 64 + j];
        const float w = sc == -INFINITY ? 0.f : exp2f(sc - m_new);
        sP[h * 64 + j] = w;
        sum += w;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0) {
        const float alpha = m_old == -INFINITY ? 0.f : exp2f(m_old - m_new);
        sA[h] = alpha;
        sM[h] = m_new;
        sL[h] = sL[h] * alpha + sum;
      }
    }
    __syncthreads();
    // this warp's share of o[h] = o[h] * alpha + sum_j p[h][j] v_j
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float al = sA[h];
#pragma unroll
      for (int k = 0; k < CPL; ++k) acc[h][k] *= al;
    }
    for (int jj = 0; jj < KPW; ++jj) {
      const int j = j0 + jj;
      const __nv_bfloat16* vr = vb + j * D + lane * CPL;
      float vf[CPL];
      if constexpr (CPL == 4) {
        const uint2 raw = *reinterpret_cast<const uint2*>(vr);
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
        const float2 y = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
        vf[0] = x.x; vf[1] = x.y; vf[2] = y.x; vf[3] = y.y;
      } else {
        const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vr));
        vf[0] = x.x; vf[1] = x.y;
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float w = sP[h * 64 + j];
#pragma unroll
        for (int k = 0; k < CPL; ++k) acc[h][k] = fmaf(w, vf[k], acc[h][k]);
      }
    }
    __syncthreads();  // the weights and this page's buffer are reused next
  }
  cp_async_wait<0>();
  // the warps' partial outputs, added in warp order
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < CPL; ++k) sO[(warp * G + h) * D + lane * CPL + k] = acc[h][k];
  __syncthreads();
  for (int x = threadIdx.x; x < G * D; x += kDecodeThreads) {
    float tot = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) tot += sO[w * G * D + x];
    a.part_o[part * G * D + x] = tot;
  }
  if (threadIdx.x < G) {
    a.part_ml[(part * G + threadIdx.x) * 2] = sM[threadIdx.x];
    a.part_ml[(part * G + threadIdx.x) * 2 + 1] = sL[threadIdx.x];
  }
}

// 2. merge the splits of one table
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_combine_kernel(const __grid_constant__ DecodeArgs a) {
  const int t = blockIdx.x;
  const int kvh = t % a.hkv, layer = (t / a.hkv) % a.n_layers, r = t / (a.hkv * a.n_layers);
  const int n_e = a.entry_count[t];
  {
    const int rc = a.range_count[t];
    if (n_e == 0 || rc == 0 || a.ranges[a.range_start[t] + rc - 1].end != a.req_len[r])
      return;  // the request's last position is not a row of this table
  }
  const int n_split = (n_e + kDecodePages - 1) / kDecodePages;
  const int64_t base = static_cast<int64_t>(t) * a.max_splits;
  for (int x = threadIdx.x; x < G * D; x += kDecodeThreads) {
    const int h = x / D, c = x % D;
    float M = -INFINITY;
    for (int s = 0; s < n_split; ++s) M = fmaxf(M, a.part_ml[((base + s) * G + h) * 2]);
    float L = 0.f, acc = 0.f;
    if (M != -INFINITY) {
      for (int s = 0; s < n_split; ++s) {
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
  const size_t smem = 4 * 64 * D * sizeof(__nv_bfloat16) +
                      (G * 64 + 3 * G + (kDecodeThreads / 32) * G * D) * sizeof(float);
  auto split = decode_split_kernel<D, G>;
  cudaError_t e = cudaFuncSetAttribute(split, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  split<<<dim3(n_tables, a.max_splits), kDecodeThreads, smem, stream>>>(a);
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
  a.max_splits = in.max_splits;
  a.window = in.window;
  a.scale_log2 = in.softmax_scale * 1.4426950408889634f;
  for (int k = 0; k < in.n_layers * in.hkv; ++k) a.cls[k] = in.cls[k];
  a.error_word = in.error_word;
  const int n_tables = in.n_req * in.n_layers * in.hkv;
  if (n_tables == 0 || in.max_splits == 0) return cudaSuccess;
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
