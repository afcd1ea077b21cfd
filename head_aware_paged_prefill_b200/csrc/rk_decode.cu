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
//      the kv head: each K and V page is staged in shared memory, the G x P
//      scores (fp32) are masked by the class rule, an online softmax per head
//      keeps (m, l) and the partial output in registers; the split writes
//      (o, m, l) to the workspace;
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

// 1. one split of one table
template <int D, int G>
__global__ void __launch_bounds__(kDecodeThreads)
    decode_split_kernel(const __grid_constant__ DecodeArgs a) {
  constexpr int NO = (G * D + kDecodeThreads - 1) / kDecodeThreads;  // outputs per thread
  extern __shared__ __align__(16) uint8_t smem[];
  const int P = a.p;
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sV = sK + 64 * D;
  float* sQ = reinterpret_cast<float*>(sV + 64 * D);  // [G][D]
  float* sP = sQ + G * D;                             // [G][64] scores, then weights
  float* sM = sP + G * 64;                            // [G] running max (log2 domain)
  float* sL = sM + G;                                 // [G] running sum
  float* sA = sL + G;                                 // [G] rescale of this page
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
  // this thread's outputs: x = threadIdx.x + 128 k, head x / D, column x % D
  float acc[NO];
#pragma unroll
  for (int k = 0; k < NO; ++k) acc[k] = 0.f;
  // the G queries, scaled into the log2 domain
  for (int x = threadIdx.x; x < G * D; x += kDecodeThreads) {
    const int h = x / D, c = x % D;
    const int64_t qi = ((static_cast<int64_t>(layer) * a.n_req + r) * a.hq + kvh * G + h) * D + c;
    sQ[x] = __bfloat162float(a.q[qi]) * a.scale_log2;
  }
  if (threadIdx.x < G) {
    sM[threadIdx.x] = -INFINITY;
    sL[threadIdx.x] = 0.f;
  }
  __syncthreads();
  const int e_end = min(n_e, e0 + kDecodePages);
  for (int e = e0; e < e_end; ++e) {
    const rk_entry en = a.entries[e_first + e];
    const bool ok_page = en.phys_page >= 0 && en.phys_page < a.n_pages;
    if (!ok_page) {
      if (threadIdx.x == 0) atomicOr(a.error_word, static_cast<int>(RK_DEV_BAD_PAGE));
      continue;  // uniform across the CTA
    }
    // stage the page's K and V (16-byte chunks)
    const uint4* gk = reinterpret_cast<const uint4*>(a.k_pool + static_cast<int64_t>(en.phys_page) * P * D);
    const uint4* gv = reinterpret_cast<const uint4*>(a.v_pool + static_cast<int64_t>(en.phys_page) * P * D);
    uint4* k4 = reinterpret_cast<uint4*>(sK);
    uint4* v4 = reinterpret_cast<uint4*>(sV);
    for (int x = threadIdx.x; x < P * D / 8; x += kDecodeThreads) {
      k4[x] = gk[x];
      v4[x] = gv[x];
    }
    __syncthreads();
    // scores s[h][j] = q_h . k_j (log2 domain), -inf where not visible; a
    // thread walks the columns from its own offset so the lanes of a warp
    // read different banks of the key row
    for (int x = threadIdx.x; x < G * P; x += kDecodeThreads) {
      const int h = x / P, j = x % P;
      const int pos = en.logical_pos + j;
      float s = -INFINITY;
      if (j < en.n_valid && pos <= row && pos >= lo) {
        const __nv_bfloat162* kr = reinterpret_cast<const __nv_bfloat162*>(sK + j * D);
        const float* qh = sQ + h * D;
        float acc0 = 0.f, acc1 = 0.f;
        const int rot = (threadIdx.x & 31) % (D / 2);
#pragma unroll 8
        for (int c2 = 0; c2 < D / 2; ++c2) {
          const int cc = (c2 + rot) % (D / 2);
          const float2 kv = __bfloat1622float2(kr[cc]);
          acc0 = fmaf(qh[2 * cc], kv.x, acc0);
          acc1 = fmaf(qh[2 * cc + 1], kv.y, acc1);
        }
        s = acc0 + acc1;
      }
      sP[h * 64 + j] = s;
    }
    __syncthreads();
    // per head (one warp each): new running max, weights p = 2^(s - m),
    // rescale factor
    for (int h = threadIdx.x >> 5; h < G; h += kDecodeThreads / 32) {
      const int lane = threadIdx.x & 31;
      float mx = -INFINITY;
      for (int j = lane; j < P; j += 32) mx = fmaxf(mx, sP[h * 64 + j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float m_old = sM[h];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int j = lane; j < P; j += 32) {
        const float s = sP[h * 64 + j];
        const float w = s == -INFINITY ? 0.f : exp2f(s - m_new);
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
    // o[h] = o[h] * alpha + sum_j p[h][j] v_j
#pragma unroll
    for (int k = 0; k < NO; ++k) {
      const int x = threadIdx.x + kDecodeThreads * k;
      if (x < G * D) {
        const int h = x / D, c = x % D;
        const float* ph = sP + h * 64;
        float v = acc[k] * sA[h];
        for (int j = 0; j < P; ++j) v = fmaf(ph[j], __bfloat162float(sV[j * D + c]), v);
        acc[k] = v;
      }
    }
    __syncthreads();  // the page buffers are refilled next
  }
#pragma unroll
  for (int k = 0; k < NO; ++k) {
    const int x = threadIdx.x + kDecodeThreads * k;
    if (x < G * D) a.part_o[part * G * D + x] = acc[k];
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
  const size_t smem = 2 * 64 * D * sizeof(__nv_bfloat16) + (G * D + G * 64 + 3 * G) * sizeof(float);
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
