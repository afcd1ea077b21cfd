// K2: RoPE relocation of cached K pages (RedKnot README excerpt, "Offline KV
// Reuse + RoPE Relocation": stored KV is re-rotated to the position it is
// reused at, which keeps it numerically aligned with online KV).
//
// Rotate-half convention: pair m = (m, m + D/2) rotates by delta * f_m with
// f_m = theta^(-2m/D).  Since R(delta) R(p) = R(p + delta), a key stored
// rotated at position p reaches position p + delta by one more rotation.
//
// HBM-bound streaming kernel.  A page is one contiguous P x D bf16 block, so
// it moves with untiled bulk copies: each CTA owns a contiguous block of jobs
// and a ring of page-sized shared-memory stages.  One thread keeps the ring
// full (bulk loads signalling a per-stage mbarrier) and drains it (bulk
// stores); all threads rotate the staged page in place.  The sin / cos of a
// delta go into a shared table, rebuilt only when the delta changes.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rk_internal.h"
#include "sm100.cuh"

namespace rk {

struct RopeFreqs {
  double f[64];  // theta^(-2m/D), m < D/2
};

constexpr int kRelocThreads = 128;
constexpr int kRelocMaxStages = 16;
constexpr int kRelocRingBytes = 48 * 1024;

// Stages for a page size: about kRelocRingBytes of ring, 2 .. kRelocMaxStages.
__host__ __device__ inline int reloc_stages(int page_bytes) {
  int s = kRelocRingBytes / page_bytes;
  return s < 2 ? 2 : (s > kRelocMaxStages ? kRelocMaxStages : s);
}

inline size_t reloc_smem_bytes(int page_bytes, int D) {
  return static_cast<size_t>(reloc_stages(page_bytes)) * page_bytes + sizeof(float2) * (D / 2) +
         sizeof(uint64_t) * kRelocMaxStages;
}

struct RelocJob {
  int src, dst, delta;
  bool valid;  // both page ids inside their pools
  bool noop;   // delta 0 onto the same page of the same pool
};

__device__ __forceinline__ RelocJob reloc_job(const int32_t* jobs, int j, int64_t n_src,
                                              int64_t n_dst, bool same_pool) {
  RelocJob r;
  r.src = jobs[3 * j];
  r.dst = jobs[3 * j + 1];
  r.delta = jobs[3 * j + 2];
  r.valid = r.src >= 0 && r.src < n_src && r.dst >= 0 && r.dst < n_dst;
  r.noop = r.delta == 0 && same_pool && r.src == r.dst;
  return r;
}

template <int D>
__global__ void __launch_bounds__(kRelocThreads)
    relocate_kernel(const __nv_bfloat16* __restrict__ src_pool, __nv_bfloat16* dst_pool,
                    const int32_t* __restrict__ jobs, int n_jobs, int P, int64_t n_src_pages,
                    int64_t n_dst_pages, const RopeFreqs freqs, int* device_error) {
  constexpr int H = D / 2;
  constexpr int VPR = H / 8;  // 16-byte vectors per half row
  extern __shared__ __align__(128) uint8_t smem[];
  const uint32_t page_bytes = static_cast<uint32_t>(P) * D * 2;
  const int S = reloc_stages(static_cast<int>(page_bytes));
  float2* cs = reinterpret_cast<float2*>(smem + static_cast<size_t>(S) * page_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(cs + H);
  const bool same_pool = static_cast<const void*>(src_pool) == static_cast<const void*>(dst_pool);

  const int per = (n_jobs + gridDim.x - 1) / gridDim.x;
  const int j_begin = blockIdx.x * per;
  const int n_my = min(per, n_jobs - j_begin);
  if (n_my <= 0) return;
  const int tid = threadIdx.x;

  // ring producer (thread 0): a job whose pages are invalid or that has
  // nothing to move still completes its stage's phase, with a plain arrive
  auto issue = [&](int i) {
    const RelocJob jb = reloc_job(jobs, j_begin + i, n_src_pages, n_dst_pages, same_pool);
    uint64_t* bar = &full[i % S];
    if (jb.valid && !jb.noop) {
      mbar_arrive_expect_tx(bar, page_bytes);
      bulk_load_g2s(smem + static_cast<size_t>(i % S) * page_bytes,
                    src_pool + static_cast<int64_t>(jb.src) * P * D, page_bytes, bar);
    } else {
      if (!jb.valid && device_error) atomicOr(device_error, static_cast<int>(RK_DEV_BAD_PAGE));
      mbar_arrive(bar);
    }
  };

  int n_issued = 0;
  if (tid == 0) {
    for (int s = 0; s < S; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    for (; n_issued < min(S, n_my); ++n_issued) issue(n_issued);
  }
  __syncthreads();

  // a thread always works on the same 16-byte column chunk of a half row
  // (kRelocThreads is a multiple of VPR), so it keeps that chunk's 8 cos /
  // sin pairs in registers, reloaded only when the table changes
  static_assert(kRelocThreads % VPR == 0, "chunk of a thread must not change");
  const int m0 = (tid % VPR) * 8;
  float2 cr[8];
  int tab_delta = 0;
  bool tab_valid = false;
  int i = 0;
  bool ok = true;
  for (; i < n_my; ++i) {
    const RelocJob jb = reloc_job(jobs, j_begin + i, n_src_pages, n_dst_pages, same_pool);
    const int stage = i % S;
    // every thread is past the previous job's rotation (the barrier before
    // its store), so the table may change; it does so while the page loads
    if (jb.valid && jb.delta != 0 && (!tab_valid || jb.delta != tab_delta)) {
      if (tid < H) {
        // angle formed and reduced modulo 2 pi in fp64 (2 pi split in a head
        // and a tail constant), sin / cos of the reduced angle in fp32
        const double a = static_cast<double>(jb.delta) * freqs.f[tid];
        const double k = rint(a * 0.15915494309189535);
        double red = fma(-k, 6.283185307179586, a);
        red = fma(-k, 2.4492935982947064e-16, red);
        float sn, cn;
        sincosf(static_cast<float>(red), &sn, &cn);
        cs[tid] = make_float2(cn, sn);
      }
      __syncthreads();
#pragma unroll
      for (int k = 0; k < 8; ++k) cr[k] = cs[m0 + k];
      tab_delta = jb.delta;
      tab_valid = true;
    }
    bool got = mbar_wait_drain(&full[stage], (i / S) & 1);
    if (!__syncthreads_and(got)) {
      ok = false;
      break;
    }
    uint4* buf = reinterpret_cast<uint4*>(smem + static_cast<size_t>(stage) * page_bytes);
    if (jb.valid && jb.delta != 0) {
      for (int v = tid; v < P * VPR; v += kRelocThreads) {
        const int idx = (v / VPR) * (D / 8) + (v % VPR);
        uint4 a = buf[idx], b = buf[idx + H / 8];
        __nv_bfloat162* a2 = reinterpret_cast<__nv_bfloat162*>(&a);
        __nv_bfloat162* b2 = reinterpret_cast<__nv_bfloat162*>(&b);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 x0 = __bfloat1622float2(a2[k]);
          const float2 x1 = __bfloat1622float2(b2[k]);
          const float2 c0 = cr[2 * k], c1 = cr[2 * k + 1];
          a2[k] = __floats2bfloat162_rn(x0.x * c0.x - x1.x * c0.y, x0.y * c1.x - x1.y * c1.y);
          b2[k] = __floats2bfloat162_rn(x0.x * c0.y + x1.x * c0.x, x0.y * c1.y + x1.y * c1.x);
        }
        buf[idx] = a;
        buf[idx + H / 8] = b;
      }
    }
    fence_proxy_async_smem();  // the rotated page is read by the bulk store
    __syncthreads();
    if (tid == 0) {
      if (jb.valid && !jb.noop)
        bulk_store_s2g(dst_pool + static_cast<int64_t>(jb.dst) * P * D, buf, page_bytes);
      bulk_commit();
      // refill the stage of the previous job once its store has read it
      if (i >= 1 && n_issued < n_my) {
        bulk_wait_read<1>();
        issue(n_issued++);
      }
    }
  }
  if (tid == 0) {
    if (!ok) {
      if (device_error) atomicOr(device_error, static_cast<int>(RK_DEV_TIMEOUT));
      // let every load still in flight land before the CTA's memory goes away
      for (int k = i; k < n_issued; ++k) mbar_wait_drain(&full[k % S], (k / S) & 1);
    }
    bulk_wait<0>();
  }
}

cudaError_t launch_relocate(const void* k_src, void* k_dst, const int32_t* jobs, int n_jobs,
                            int64_t n_src_pages, int64_t n_dst_pages, int P, int D, double theta,
                            int* device_error, cudaStream_t stream) {
  if (n_jobs == 0) return cudaSuccess;
  RopeFreqs f;
  for (int m = 0; m < D / 2; ++m) f.f[m] = pow(theta, -2.0 * m / D);
  const int page_bytes = P * D * 2;
  const size_t smem = reloc_smem_bytes(page_bytes, D);
  auto kern = D == 128 ? relocate_kernel<128> : relocate_kernel<64>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kRelocThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int grid = n_jobs < sms * per_sm ? n_jobs : sms * per_sm;
  kern<<<grid, kRelocThreads, smem, stream>>>(
      static_cast<const __nv_bfloat16*>(k_src), static_cast<__nv_bfloat16*>(k_dst), jobs, n_jobs,
      P, n_src_pages, n_dst_pages, f, device_error);
  return cudaGetLastError();
}

}  // namespace rk
