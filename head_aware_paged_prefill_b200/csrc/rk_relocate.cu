// K2: RoPE relocation of cached K pages (RedKnot README excerpt, "Offline KV
// Reuse + RoPE Relocation": stored KV is re-rotated to the position it is
// reused at, which keeps it numerically aligned with online KV).
//
// Rotate-half convention: pair m = (m, m + D/2) rotates by delta * f_m with
// f_m = theta^(-2m/D).  Since R(delta) R(p) = R(p + delta), a key stored
// rotated at position p reaches position p + delta by one more rotation.
//
// HBM-bound streaming kernel: one CTA per page job, each thread moves 16-byte
// vectors of both halves of a row, angles are formed and reduced in fp64 and
// their sin / cos evaluated once per job into shared memory.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rk_internal.h"

namespace rk {

struct RopeFreqs {
  double f[64];  // theta^(-2m/D), m < D/2
};

constexpr int kRelocThreads = 256;

template <int D>
__global__ void __launch_bounds__(kRelocThreads)
    relocate_kernel(const __nv_bfloat16* __restrict__ src_pool, __nv_bfloat16* __restrict__ dst_pool,
                    const int32_t* __restrict__ jobs, int n_jobs, int P, int64_t n_pages,
                    const RopeFreqs freqs, int* device_error) {
  constexpr int H = D / 2;
  constexpr int VPR = H / 8;  // 16-byte vectors per half row
  __shared__ float2 cs[H];
  for (int job = blockIdx.x; job < n_jobs; job += gridDim.x) {
    const int src = jobs[3 * job], dst = jobs[3 * job + 1], delta = jobs[3 * job + 2];
    if (src < 0 || src >= n_pages || dst < 0 || dst >= n_pages) {
      if (threadIdx.x == 0 && device_error) atomicOr(device_error, static_cast<int>(RK_DEV_BAD_PAGE));
      continue;
    }
    const uint4* s = reinterpret_cast<const uint4*>(src_pool + static_cast<int64_t>(src) * P * D);
    uint4* d = reinterpret_cast<uint4*>(dst_pool + static_cast<int64_t>(dst) * P * D);
    if (delta == 0) {
      if (src != dst) {
        for (int v = threadIdx.x; v < P * D / 8; v += kRelocThreads) d[v] = s[v];
      }
      continue;
    }
    __syncthreads();  // previous job's readers of cs are done
    if (threadIdx.x < H) {
      double sn, cn;
      sincos(static_cast<double>(delta) * freqs.f[threadIdx.x], &sn, &cn);
      cs[threadIdx.x] = make_float2(static_cast<float>(cn), static_cast<float>(sn));
    }
    __syncthreads();
    for (int v = threadIdx.x; v < P * VPR; v += kRelocThreads) {
      const int row = v / VPR, m0 = (v % VPR) * 8;
      const uint4 a = s[(row * D + m0) / 8];
      const uint4 b = s[(row * D + H + m0) / 8];
      const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
      const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
      uint4 oa, ob;
      __nv_bfloat162* oa2 = reinterpret_cast<__nv_bfloat162*>(&oa);
      __nv_bfloat162* ob2 = reinterpret_cast<__nv_bfloat162*>(&ob);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float2 x0 = __bfloat1622float2(a2[k]);
        const float2 x1 = __bfloat1622float2(b2[k]);
        const float2 c0 = cs[m0 + 2 * k], c1 = cs[m0 + 2 * k + 1];
        const float y0a = x0.x * c0.x - x1.x * c0.y;
        const float y1a = x0.x * c0.y + x1.x * c0.x;
        const float y0b = x0.y * c1.x - x1.y * c1.y;
        const float y1b = x0.y * c1.y + x1.y * c1.x;
        oa2[k] = __floats2bfloat162_rn(y0a, y0b);
        ob2[k] = __floats2bfloat162_rn(y1a, y1b);
      }
      d[(row * D + m0) / 8] = oa;
      d[(row * D + H + m0) / 8] = ob;
    }
  }
}

cudaError_t launch_relocate(const void* k_src, void* k_dst, const int32_t* jobs, int n_jobs,
                            int64_t n_pages, int P, int D, double theta, int* device_error,
                            cudaStream_t stream) {
  if (n_jobs == 0) return cudaSuccess;
  RopeFreqs f;
  for (int m = 0; m < D / 2; ++m) f.f[m] = pow(theta, -2.0 * m / D);
  const int grid = n_jobs < (1 << 30) ? n_jobs : (1 << 30);
  if (D == 128) {
    relocate_kernel<128><<<grid, kRelocThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_src), static_cast<__nv_bfloat16*>(k_dst), jobs,
        n_jobs, P, n_pages, f, device_error);
  } else {
    relocate_kernel<64><<<grid, kRelocThreads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(k_src), static_cast<__nv_bfloat16*>(k_dst), jobs,
        n_jobs, P, n_pages, f, device_error);
  }
  return cudaGetLastError();
}

}  // namespace rk
