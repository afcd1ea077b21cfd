// K2: RoPE relocation of cached K pages (RedKnot README excerpt, "Offline KV
// Reuse + RoPE Relocation": stored KV is re-rotated to the position it is
// reused at, which keeps it numerically aligned with online KV).
//
// Rotate-half convention: pair m = (m, m + D/2) rotates by delta * f_m with
// f_m = theta^(-2m/D).  Since R(delta) R(p) = R(p + delta), a key stored
// rotated at position p reaches position p + delta by one more rotation.
//
// HBM-bound streaming kernel: each thread moves 16-byte vectors of both
// halves of a row; the sin / cos of a delta are evaluated in fp64 into a
// shared table that consecutive jobs with the same delta reuse.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rk_internal.h"

namespace rk {

struct RopeFreqs {
  double f[64];  // theta^(-2m/D), m < D/2
};

constexpr int kRelocThreads = 256;

// Each CTA takes a contiguous block of jobs (a relocation plan lists the pages
// of one segment, which share a delta, one after another).  Per job, every
// thread first issues its 16-byte loads (both rotate-half partners of its
// chunks), then the cos / sin table is rebuilt only if the delta changed, so
// the table's fp64 work overlaps the loads in flight.
template <int D>
__global__ void __launch_bounds__(kRelocThreads)
    relocate_kernel(const __nv_bfloat16* __restrict__ src_pool, __nv_bfloat16* __restrict__ dst_pool,
                    const int32_t* __restrict__ jobs, int n_jobs, int P, int64_t n_src_pages,
                    int64_t n_dst_pages, const RopeFreqs freqs, int* device_error) {
  constexpr int H = D / 2;
  constexpr int VPR = H / 8;  // 16-byte vectors per half row
  constexpr int NV = 2;       // vector pairs per thread per pass
  __shared__ float2 cs[H];
  const int per = (n_jobs + gridDim.x - 1) / gridDim.x;
  const int j_begin = blockIdx.x * per;
  const int j_end = min(j_begin + per, n_jobs);
  int tab_delta = 0;
  bool tab_valid = false;
  for (int job = j_begin; job < j_end; ++job) {
    const int src = jobs[3 * job], dst = jobs[3 * job + 1], delta = jobs[3 * job + 2];
    if (src < 0 || src >= n_src_pages || dst < 0 || dst >= n_dst_pages) {
      if (threadIdx.x == 0 && device_error) atomicOr(device_error, static_cast<int>(RK_DEV_BAD_PAGE));
      continue;
    }
    const uint4* sp = reinterpret_cast<const uint4*>(src_pool + static_cast<int64_t>(src) * P * D);
    uint4* dp = reinterpret_cast<uint4*>(dst_pool + static_cast<int64_t>(dst) * P * D);
    if (delta == 0) {
      if (sp != dp) {
        for (int v = threadIdx.x; v < P * D / 8; v += kRelocThreads) dp[v] = sp[v];
      }
      continue;
    }
    for (int base = 0; base < P * VPR; base += NV * kRelocThreads) {
      uint4 a[NV], bq[NV];
      int idx[NV];
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        const int v = base + u * kRelocThreads + threadIdx.x;
        idx[u] = v < P * VPR ? (v / VPR) * (D / 8) + (v % VPR) : -1;
        if (idx[u] >= 0) {
          a[u] = sp[idx[u]];
          bq[u] = sp[idx[u] + H / 8];
        }
      }
      if (base == 0 && (!tab_valid || delta != tab_delta)) {
        __syncthreads();  // every thread is done with the previous table
        if (threadIdx.x < H) {
          double sn, cn;
          sincos(static_cast<double>(delta) * freqs.f[threadIdx.x], &sn, &cn);
          cs[threadIdx.x] = make_float2(static_cast<float>(cn), static_cast<float>(sn));
        }
        __syncthreads();
        tab_delta = delta;
        tab_valid = true;
      }
#pragma unroll
      for (int u = 0; u < NV; ++u) {
        if (idx[u] < 0) continue;
        const int m0 = (idx[u] % (D / 8)) * 8;
        __nv_bfloat162* a2 = reinterpret_cast<__nv_bfloat162*>(&a[u]);
        __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&bq[u]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 x0 = __bfloat1622float2(a2[k]);
          const float2 x1 = __bfloat1622float2(b2[k]);
          const float2 c0 = cs[m0 + 2 * k], c1 = cs[m0 + 2 * k + 1];
          a2[k] = __floats2bfloat162_rn(x0.x * c0.x - x1.x * c0.y, x0.y * c1.x - x1.y * c1.y);
          b2[k] = __floats2bfloat162_rn(x0.x * c0.y + x1.x * c0.x, x0.y * c1.y + x1.y * c1.x);
        }
        dp[idx[u]] = a[u];
        dp[idx[u] + H / 8] = bq[u];
      }
    }
  }
}

cudaError_t launch_relocate(const void* k_src, void* k_dst, const int32_t* jobs, int n_jobs,
                            int64_t n_src_pages, int64_t n_dst_pages, int P, int D, double theta,
                            int* device_error, cudaStream_t stream) {
  if (n_jobs == 0) return cudaSuccess;
  RopeFreqs f;
  for (int m = 0; m < D / 2; ++m) f.f[m] = pow(theta, -2.0 * m / D);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = n_jobs < 8 * sms ? n_jobs : 8 * sms;
  if (D == 128) {
    relocate_kernel<128><<<grid, kRelocThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_src), static_cast<__nv_bfloat16*>(k_dst), jobs,
        n_jobs, P, n_src_pages, n_dst_pages, f, device_error);
  } else {
    relocate_kernel<64><<<grid, kRelocThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_src), static_cast<__nv_bfloat16*>(k_dst), jobs,
        n_jobs, P, n_src_pages, n_dst_pages, f, device_error);
  }
  return cudaGetLastError();
}

}  // namespace rk
