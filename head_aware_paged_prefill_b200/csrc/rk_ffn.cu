// Token-selective FFN: the tokens the attention importance picked run the
// layer's FFN, every other token keeps its hidden state (the residual path).
// README "About" (Elastic Sparsity / Sparse FFN) and the paooo page ("main
// functions") state the idea; the pages name the Mistral-7B and Qwen3
// families, whose FFN is the gated SiLU MLP, so for a selected row i:
//   h = silu(W_gate x_i) * (W_up x_i),   x_i <- x_i + W_down h.
//
// Three launches:
//   1. gather: the selected rows of x into a packed [M][d_model] matrix (and
//      their row ids), M = the selection's size;
//   2. GEMM 1: [M][d_model] x [2 d_ff][d_model]^T on the tensor cores, the
//      gate and up rows of one 128-wide slice of d_ff side by side in one
//      N = 256 B tile; the epilogue forms silu(g) * u and writes H [M][d_ff]
//      in bf16;
//   3. GEMM 2: H x W_down^T, N = 256 columns of d_model per tile; the
//      epilogue adds the product to x at the selected row (in place).
// The GEMM is persistent (one CTA per SM) and warp-specialised: warp 0
// issues TMA loads of A (128 x 64) and B (256 x 64) tiles into a four-stage
// ring, warp 1 issues tcgen05.mma (M 128, N 256, K 16) into one of two TMEM
// accumulators, warps 2-5 drain the other accumulator through the epilogue,
// so the epilogue of one tile overlaps the main loop of the next.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "rk_internal.h"
#include "sm100.cuh"

namespace rk {

namespace {

constexpr int kFfnThreads = 192;  // producer, MMA issuer, 4 epilogue warps
constexpr int kFfnStages = 4;
constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kABytes = kBM * kBK * 2;  // 16 KB
constexpr int kBBytes = kBN * kBK * 2;  // 32 KB
constexpr int kStageBytes = kABytes + kBBytes;
constexpr int kFfnSmem = kFfnStages * kStageBytes + 256 + 1024;
constexpr int kGroupM = 16;  // m-blocks per rasterisation group (L2 reuse of A and B)

enum FfnEpi : int { kEpiSwiGLU = 0, kEpiResidual = 1 };

struct GemmParams {
  int m, n_tiles_n, k_steps;  // rows, tiles along N, K / 64
  // kEpiSwiGLU: out = H [m][ld_out], the tile's 128 outputs at n_blk * 128
  // kEpiResidual: x [.][ld_out] += acc at row rows[m], columns n_blk * 256
  __nv_bfloat16* out;
  int ld_out;
  const int32_t* rows;
  int32_t* error_word;
  int* timeout_site;
  int b1_row_offset;  // row of the second 128-row B box relative to the first's
  int b_row_step;     // B rows per n-block (128 for gate/up, 256 for down)
};

__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fdividef(g, 1.0f + __expf(-g)) * u;
}

template <int EPI>
__global__ void __launch_bounds__(kFfnThreads, 1)
    ffn_gemm_kernel(const __grid_constant__ CUtensorMap tm_a,
                    const __grid_constant__ CUtensorMap tm_b0,
                    const __grid_constant__ CUtensorMap tm_b1,
                    const __grid_constant__ GemmParams prm) {
  extern __shared__ uint8_t ffn_raw[];
  uint8_t* sm = ffn_raw + ((1024 - (smem_u32(ffn_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kFfnStages * kStageBytes);
  uint64_t* full = bars;                    // [kFfnStages] TMA bytes
  uint64_t* empty = bars + kFfnStages;      // [kFfnStages] tcgen05.commit
  uint64_t* acc_full = bars + 2 * kFfnStages;      // [2] tcgen05.commit
  uint64_t* acc_empty = bars + 2 * kFfnStages + 2;  // [2] 128 epilogue threads
  uint64_t* drain = bars + 2 * kFfnStages + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kFfnStages + 5);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kFfnStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b0);
    prefetch_tensormap(&tm_b1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtx wc{abort_flag, prm.error_word, prm.timeout_site};
  const int n_mblk = (prm.m + kBM - 1) / kBM;
  const int n_tiles = n_mblk * prm.n_tiles_n;
  // tile -> (m block, n block): m fastest inside groups of kGroupM m-blocks
  auto tile_mn = [&](int t, int& mb, int& nb) {
    const int per_group = kGroupM * prm.n_tiles_n;
    const int g = t / per_group, rem = t % per_group;
    const int gm = min(kGroupM, n_mblk - g * kGroupM);
    mb = g * kGroupM + rem % gm;
    nb = rem / gm;
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
        int mb, nb;
        tile_mn(t, mb, nb);
        const int b_row = nb * prm.b_row_step;
        for (int k = 0; k < prm.k_steps; ++k, ++it) {
          const int s = it % kFfnStages;
          if (it >= kFfnStages &&
              !(ok = mbar_wait(&empty[s], ((it / kFfnStages) - 1) & 1, wc, 1)))
            break;
          uint8_t* st = sm + s * kStageBytes;
          mbar_arrive_expect_tx(&full[s], kStageBytes);
          tma_load_2d(st, &tm_a, &full[s], k * kBK, mb * kBM);
          tma_load_2d(st + kABytes, &tm_b0, &full[s], k * kBK, b_row);
          tma_load_2d(st + kABytes + kBBytes / 2, &tm_b1, &full[s], k * kBK,
                      b_row + prm.b1_row_offset);
        }
      }
      // loads in flight after an abort land before the CTA leaves
      for (uint32_t x = it > kFfnStages ? it - kFfnStages : 0; x < it; ++x)
        mbar_wait_drain(&full[x % kFfnStages], (x / kFfnStages) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, false);
      const uint32_t s_u = smem_u32(sm);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++tc) {
        const int buf = tc & 1;
        if (tc >= 2 && !(ok = mbar_wait(&acc_empty[buf], ((tc >> 1) - 1) & 1, wc, 2))) break;
        tc_fence_after();
        for (int k = 0; k < prm.k_steps; ++k, ++it) {
          const int s = it % kFfnStages;
          if (!(ok = mbar_wait(&full[s], (it / kFfnStages) & 1, wc, 3))) break;
          tc_fence_after();
          const uint32_t a0 = s_u + s * kStageBytes, b0 = a0 + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_ss(tmem + buf * kBN, desc_sw128(a0 + kk * 32, 16, 1024),
                        desc_sw128(b0 + kk * 32, 16, 1024), idesc, (k | kk) ? 1u : 0u);
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
      }
      tc_commit(drain);
      mbar_wait_drain(drain, 0);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row_in_tile = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t tc = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++tc) {
      const int buf = tc & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[buf], (tc >> 1) & 1, wc, 4));
      if (!ok) break;
      tc_fence_after();
      int mb, nb;
      tile_mn(t, mb, nb);
      const int m = mb * kBM + row_in_tile;
      const bool live = m < prm.m;
      const uint32_t ta = tmem + lane_base + buf * kBN;
      if (EPI == kEpiSwiGLU) {
        __nv_bfloat16* dst = prm.out + static_cast<int64_t>(m) * prm.ld_out + nb * 128;
#pragma unroll 1
        for (int c = 0; c < 128; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld_x32(ta + c, g);
          tmem_ld_x32(ta + 128 + c, u);
          tmem_ld_wait(g);
          tmem_ld_wait(u);
          if (live) {
            uint32_t packed[16];
#pragma unroll
            for (int j = 0; j < 16; ++j)
              packed[j] = pack_bf16x2(silu_mul(__uint_as_float(g[2 * j]), __uint_as_float(u[2 * j])),
                                      silu_mul(__uint_as_float(g[2 * j + 1]),
                                               __uint_as_float(u[2 * j + 1])));
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              d4[j] = make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
        }
      } else {
        const int row = live ? prm.rows[m] : -1;
        __nv_bfloat16* dst = prm.out + static_cast<int64_t>(row) * prm.ld_out + nb * kBN;
#pragma unroll 1
        for (int c = 0; c < kBN; c += 32) {
          uint32_t v[32];
          tmem_ld_x32(ta + c, v);
          tmem_ld_wait(v);
          if (row >= 0) {
            uint4* d4 = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              uint4 xv = d4[j];
              uint32_t* xw = reinterpret_cast<uint32_t*>(&xv);
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float lo = __uint_as_float(xw[q] << 16) + __uint_as_float(v[8 * j + 2 * q]);
                const float hi =
                    __uint_as_float(xw[q] & 0xFFFF0000u) + __uint_as_float(v[8 * j + 2 * q + 1]);
                xw[q] = pack_bf16x2(lo, hi);
              }
              d4[j] = xv;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The selected rows: selection entry m of request r (the first
// min(top_k, L_r) picks of each request, in order) is row cu[r] + token.
__global__ void __launch_bounds__(256)
    ffn_gather_kernel(const __nv_bfloat16* __restrict__ x, int d_model,
                      const int32_t* __restrict__ cu, const int32_t* __restrict__ sel_prefix,
                      int n_req, const int32_t* __restrict__ tokens, int top_k,
                      __nv_bfloat16* __restrict__ xs, int32_t* __restrict__ rows,
                      int32_t* error_word) {
  const int m = blockIdx.x;
  int lo = 0, hi = n_req;  // last r with sel_prefix[r] <= m
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sel_prefix[mid] <= m) lo = mid; else hi = mid;
  }
  const int r = lo;
  const int tok = tokens[static_cast<int64_t>(r) * top_k + (m - sel_prefix[r])];
  const int L = cu[r + 1] - cu[r];
  const bool ok = tok >= 0 && tok < L;
  const int row = ok ? cu[r] + tok : -1;
  if (threadIdx.x == 0) {
    rows[m] = row;
    if (!ok) atomicOr(error_word, static_cast<int>(RK_DEV_BAD_PAGE));
  }
  const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<int64_t>(ok ? row : 0) * d_model);
  uint4* dst = reinterpret_cast<uint4*>(xs + static_cast<int64_t>(m) * d_model);
  for (int c = threadIdx.x; c < d_model / 8; c += blockDim.x)
    dst[c] = ok ? src[c] : make_uint4(0u, 0u, 0u, 0u);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn ffn_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// A row-major bf16 matrix [rows][cols] read in (64 columns x 128 rows) boxes
// with 128-byte swizzle; rows past the end read as zeros.
bool ffn_map(EncodeTiledFn enc, CUtensorMap* tm, const void* base, int64_t rows, int64_t cols) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {64, 128};
  const cuuint32_t es[2] = {1, 1};
  return enc(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_sparse_ffn(const FfnLaunchArgs& a, cudaStream_t stream) {
  if (a.m <= 0) return cudaSuccess;
  EncodeTiledFn enc = ffn_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  auto* xs = static_cast<__nv_bfloat16*>(a.xs);
  auto* h = static_cast<__nv_bfloat16*>(a.h);
  auto* x = static_cast<__nv_bfloat16*>(a.x);
  ffn_gather_kernel<<<a.m, 256, 0, stream>>>(x, a.d_model, a.cu, a.sel_prefix, a.n_req, a.tokens,
                                             a.top_k, xs, a.rows, a.error_word);
  CUtensorMap ta, tg, tu, th, td;
  if (!ffn_map(enc, &ta, xs, a.m, a.d_model) || !ffn_map(enc, &tg, a.w_gate, a.d_ff, a.d_model) ||
      !ffn_map(enc, &tu, a.w_up, a.d_ff, a.d_model) || !ffn_map(enc, &th, h, a.m, a.d_ff) ||
      !ffn_map(enc, &td, a.w_down, a.d_model, a.d_ff))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(ffn_gemm_kernel<kEpiSwiGLU>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kFfnSmem)) != cudaSuccess ||
      (e = cudaFuncSetAttribute(ffn_gemm_kernel<kEpiResidual>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kFfnSmem)) != cudaSuccess)
    return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  const int n_mblk = (a.m + kBM - 1) / kBM;
  GemmParams p1{};
  p1.m = a.m;
  p1.n_tiles_n = a.d_ff / 128;
  p1.k_steps = a.d_model / kBK;
  p1.out = h;
  p1.ld_out = a.d_ff;
  p1.rows = a.rows;
  p1.error_word = a.error_word;
  p1.timeout_site = a.timeout_site;
  p1.b1_row_offset = 0;  // the up rows of the same slice, from the up matrix
  p1.b_row_step = 128;
  const int t1 = n_mblk * p1.n_tiles_n;
  ffn_gemm_kernel<kEpiSwiGLU><<<t1 < sms ? t1 : sms, kFfnThreads, kFfnSmem, stream>>>(ta, tg, tu, p1);
  GemmParams p2 = p1;
  p2.n_tiles_n = a.d_model / kBN;
  p2.k_steps = a.d_ff / kBK;
  p2.out = x;
  p2.ld_out = a.d_model;
  p2.b1_row_offset = 128;  // rows 128..255 of the 256-row slice of W_down
  p2.b_row_step = kBN;
  const int t2 = n_mblk * p2.n_tiles_n;
  ffn_gemm_kernel<kEpiResidual><<<t2 < sms ? t2 : sms, kFfnThreads, kFfnSmem, stream>>>(th, td, td, p2);
  return cudaGetLastError();
}

}  // namespace rk
