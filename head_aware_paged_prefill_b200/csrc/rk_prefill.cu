// K3: SegPagedAttention prefill on sm_100a.
//
// RedKnot (paooo page, "technical principles"): KV is stored per head in
// pages and a fused varlen kernel attends over exactly the pages each head
// may see, with no attn_mask; global heads recompute every row causally,
// local heads compute the uncached rows over a window of reused KV (README
// excerpt, "Head Classification" and "SegPagedAttention Runtime").  Cached
// keys are re-rotated to their reuse position while they are loaded ("Offline
// KV Reuse + RoPE Relocation").
//
// One CTA per SM, persistent over the work list of rk_select_visible.  A work
// item is <= 128 rows of one request and up to two q heads of the same kv
// head: both heads see identical pages, so each K/V tile loaded into shared
// memory feeds two Q tiles.  Items arrive sorted by cost; CTA b takes item
// b, then 2G-1-b, 2G+b, ... (G = grid size), which evens out the per-SM work.
//
//   warp 0      TMA producer: Q tiles (3-D box out of [rows][Hq][D]) and, per
//               KV tile, one box per page and 64-column block out of the pool.
//   warps 1, 3  tcgen05 issuers, one per Q tile (warp 1 also owns TMEM).
//               S_t = Q_t K^T (M=128, N=128, K=D) into ONE S buffer shared by
//               both tiles: a softmax copies S to registers as soon as it
//               lands, so the next S (of the other tile) can follow at once,
//               while P_t (bf16) goes to its own 64 TMEM columns.  O_t += P_t V
//               (M=128, N=D, K=128) with P_t read from TMEM and V from shared
//               memory (MN-major operand).  Per KV tile j issuer t puts
//               S_t(j + 1) in the buffer, then issues PV_t(j).
//   warp 2      RoPE relocation (fuse_rope): rotates the Q tiles by -delta
//               once per run of tiles sharing a delta, and the K pages of a
//               tile that mixes deltas by their difference.
//   warps 4-7   softmax warpgroup of Q tile 0, warps 8-11 of Q tile 1: one
//               TMEM lane (= one query row) per thread; online softmax in the
//               log2 domain, O rescaled in TMEM only when the running max
//               grows by more than 2^8 (after the previous PV completed), P
//               stored as bf16 in 16-column quarters.  The two warpgroups
//               run free: their exponential phases overlap wherever their
//               dependencies allow (taking turns on the MUFU was slower).
// Registers are rebalanced with setmaxnreg: the first warpgroup keeps 80 per
// thread, the two softmax warpgroups get 208.
//
// Invisible pages are never loaded: the item's entry range already excludes
// them.  Element masks are evaluated only on tiles that straddle the causal
// diagonal, a window start or a partial page.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "rk_internal.h"
#include "sm100.cuh"

namespace rk {
constexpr int kPrefillThreads = 384;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint32_t kRegsAux = 80;       // warps 0-3
constexpr uint32_t kRegsSoftmax = 208;  // warps 4-11
static_assert(128 * kRegsAux + 256 * kRegsSoftmax <= 384 * 168, "register split over budget");

template <int D, int P>
struct PrefillCfg {
  static constexpr int KB = D / 64;  // 128-byte column blocks of a row
  static constexpr int kQTileBytes = kRowsPerTile * D * 2;
  static constexpr int kKVTileBytes = kKeysPerTile * D * 2;
  static constexpr int kBlockBytes = kKeysPerTile * 128;  // one column block of a tile
  // K gets one stage more than V at D = 128: the next S needs its K tile a
  // whole softmax phase earlier than the PV needs its V tile
  static constexpr int kKStages = D == 128 ? 3 : 4;
  static constexpr int kVStages = D == 128 ? 2 : 4;
  static constexpr int EPT = kKeysPerTile / P;  // pages per KV tile
  static constexpr int kDataBytes = 2 * kQTileBytes + (kKStages + kVStages) * kKVTileBytes;
  static constexpr int kSmemBytes = kDataBytes + 1024 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  // TMEM columns: O_t at 128 t, one S buffer (fp32) shared by both Q tiles
  // at 256 (a softmax copies S to registers as soon as it lands, so the
  // other tile's S can follow), and P_t (bf16, 128 keys) at 384 + 64 t
  __host__ __device__ static constexpr uint32_t col_o(int t) { return 128u * t; }
  static constexpr uint32_t kColS = 256;
  __host__ __device__ static constexpr uint32_t col_p(int t) { return 384u + 64u * t; }
};

struct PrefillParams {
  const Item* items;
  const int32_t* n_items;
  int* work_next;  // next item of the cost-sorted list to hand out
  int* work_done;  // CTAs finished
  int* error_word;
  int* timeout_site;
  const rk_entry* entries;
  __nv_bfloat16* o;
  float* lse;
  int hq;
  int total_tokens;
  int64_t n_pages;
  float scale_log2;
  int fuse_rope;
  double inv_freq[64];  // theta^(-2m/D), m < D/2
};

// barrier slots
enum : int {
  kBarQFull = 0,
  kBarQEmpty = 1,
  kBarSFull = 2,    // [2] S of Q tile t computed
  kBarSFree = 4,    // [2] S buffer read; the next S is issuer t's (one phase per S of t)
  kBarP = 6,        // [2] P of Q tile t stored
  kBarPVDone = 8,   // [2] each PV of Q tile t completed (P_t and O_t reusable)
  kBarOFull = 10,   // [2]
  kBarOEmpty = 12,  // [2]
  kBarDrain = 14,   // [2] MMA completion before TMEM is released (one per issuer)
  kBarQReady = 16,   // fused: the Q tiles hold the rotation the next S needs
  kBarQFree = 17,    // fused: every S reading the current Q rotation completed
  kBarQReload = 18,  // fused: original Q re-fetched for a new rotation
  // 19, 20 unused
  kBarItemFull = 21,   // [2] ring of work-item indices: slot written by the producer
  kBarItemEmpty = 23,  // [2] slot read by every other role
  kBarKFull = 25,  // k_full, k_ready, k_empty [kKStages] each, then v_full, v_empty [kVStages]
};

// Index of the r-th work item of this CTA, from the producer's two-slot ring
// (-1 once the list is exhausted).  Every thread of a consuming role reads
// the slot and arrives on its empty barrier.
__device__ __forceinline__ int next_item(uint64_t* bars, const volatile int* s_item, uint32_t r,
                                         const WaitCtx& wc, int site, bool& ok) {
  const int slot = r & 1;
  if (!(ok = mbar_wait(&bars[kBarItemFull + slot], (r >> 1) & 1, wc, site))) return -1;
  const int it = s_item[slot];
  mbar_arrive(&bars[kBarItemEmpty + slot]);
  return it;
}

// cos / sin of delta * f_m for the 8 frequencies m = 8c .. 8c+7 a thread
// owns, as packed pairs (m, m+1): the angle is formed and reduced modulo 2 pi
// in fp64 (2 pi split in a head and a tail constant), sin / cos in fp32.
__device__ __forceinline__ void rope_table(int delta, int c, const double* inv_freq,
                                           uint64_t (&cos2)[4], uint64_t (&sin2)[4]) {
#pragma unroll
  for (int q = 0; q < 8; q += 2) {
    float cs[2], sn[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const double a = static_cast<double>(delta) * inv_freq[8 * c + q + u];
      const double k = rint(a * 0.15915494309189535);
      double red = fma(-k, 6.283185307179586, a);
      red = fma(-k, 2.4492935982947064e-16, red);
      sincosf(static_cast<float>(red), &sn[u], &cs[u]);
    }
    cos2[q / 2] = f2_pack(cs[0], cs[1]);
    sin2[q / 2] = f2_pack(sn[0], sn[1]);
  }
}

// Rotates rows [row_lo, row_hi) of a 128-row bf16 tile in shared memory (the
// K or Q operand layout: 64-column blocks of 128-byte rows, 128-byte swizzle,
// so 16-byte chunk c of row r sits at chunk c ^ (r & 7)).  Thread rt of 32
// owns chunk c of rows r0, r0 + RSTEP, ...; the rotate-half partner of chunk c
// is chunk c + D/16 of the same row (D = 64) or chunk c of the next column
// block (D = 128).  Packed fp32 math, one bf16 rounding per element.
template <int D>
__device__ __forceinline__ void rope_rotate_rows(uint8_t* tile, int row_lo, int row_hi, int rt,
                                                 const uint64_t (&cos2)[4],
                                                 const uint64_t (&sin2)[4]) {
  constexpr int CH = D / 16;
  constexpr int RSTEP = 32 / CH;
  const int c = rt % CH;
  const int first = row_lo + ((rt / CH) - row_lo % RSTEP + RSTEP) % RSTEP;
#pragma unroll 2
  for (int r = first; r < row_hi; r += RSTEP) {
    const int sw = r & 7;
    uint8_t* row = tile + r * 128;
    uint4* plo = reinterpret_cast<uint4*>(row + ((c ^ sw) << 4));
    uint4* phi = D == 128 ? reinterpret_cast<uint4*>(row + kKeysPerTile * 128 + ((c ^ sw) << 4))
                          : reinterpret_cast<uint4*>(row + (((c + CH) ^ sw) << 4));
    uint4 a = *plo, bq = *phi;
    const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
    const uint32_t* bw = reinterpret_cast<const uint32_t*>(&bq);
    uint32_t ya[4], yb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // x0 = (x_m, x_m+1), x1 = (x_{m+D/2}, x_{m+1+D/2})
      const uint64_t x0 = f2_pack(__uint_as_float(aw[k] << 16), __uint_as_float(aw[k] & 0xFFFF0000u));
      const uint64_t x1 = f2_pack(__uint_as_float(bw[k] << 16), __uint_as_float(bw[k] & 0xFFFF0000u));
      // y0 = x0 cos - x1 sin ; y1 = x0 sin + x1 cos
      const uint64_t y0 = f2_fma(x0, cos2[k], f2_mul_neg(x1, sin2[k]));
      const uint64_t y1 = f2_fma(x0, sin2[k], f2_mul(x1, cos2[k]));
      float lo, hi;
      f2_unpack(y0, lo, hi);
      ya[k] = pack_bf16x2(lo, hi);
      f2_unpack(y1, lo, hi);
      yb[k] = pack_bf16x2(lo, hi);
    }
    *plo = make_uint4(ya[0], ya[1], ya[2], ya[3]);
    *phi = make_uint4(yb[0], yb[1], yb[2], yb[3]);
  }
}

template <int D, int P>
__global__ void __launch_bounds__(kPrefillThreads, 1)
    segpaged_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v,
                            const __grid_constant__ PrefillParams prm) {
  using C = PrefillCfg<D, P>;
  constexpr int SK = C::kKStages, SV = C::kVStages;
  static_assert(kBarKFull + 3 * SK + 2 * SV <= 64, "barrier slots");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + 2 * C::kQTileBytes;
  uint8_t* sV = sK + SK * C::kKVTileBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + SV * C::kKVTileBytes);
  uint64_t* k_full = bars + kBarKFull;
  uint64_t* k_ready = k_full + SK;
  uint64_t* k_empty = k_ready + SK;
  uint64_t* v_full = k_empty + SK;
  uint64_t* v_empty = v_full + SV;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 64);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* s_item = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [2]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool fuse = prm.fuse_rope != 0;

  if (threadIdx.x == 0) {
    // counts: 1 = one elected thread (or a tcgen05.commit), 2 = both
    // issuers, 32 = the RoPE warp, 128 = a softmax warpgroup
    mbar_init(&bars[kBarQFull], 1);
    mbar_init(&bars[kBarQEmpty], 2);
    mbar_init(&bars[kBarDrain], 1);
    mbar_init(&bars[kBarDrain + 1], 1);
    mbar_init(&bars[kBarQReady], 32);
    mbar_init(&bars[kBarQFree], 2);
    mbar_init(&bars[kBarQReload], 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bars[kBarItemFull + t], 1);
      // readers of a slot: both issuers, the RoPE warp when it runs, both
      // softmax warpgroups
      mbar_init(&bars[kBarItemEmpty + t], 2 + (fuse ? 32 : 0) + 256);
      mbar_init(&bars[kBarSFree + t], 128);
      mbar_init(&bars[kBarSFull + t], 1);
      mbar_init(&bars[kBarP + t], 128);
      mbar_init(&bars[kBarPVDone + t], 1);
      mbar_init(&bars[kBarOFull + t], 1);
      mbar_init(&bars[kBarOEmpty + t], 128);
    }
    for (int s = 0; s < SK; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_ready[s], 32);
      mbar_init(&k_empty[s], 2);
    }
    for (int s = 0; s < SV; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 2);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_q);
    prefetch_tensormap(&tm_k);
    prefetch_tensormap(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_items = *prm.n_items;
  const WaitCtx wc{abort_flag, prm.error_word, prm.timeout_site};

  if (warp < 4) {
    // The register split happens inside each role's branch so that no control
    // flow merges between setmaxnreg and the code it budgets for.
    setmaxnreg_dec<kRegsAux>();
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t k_issued = 0, v_issued = 0, q_uses = 0;
      bool ok = true;
      const int32_t oob_row = static_cast<int32_t>(prm.n_pages * P);
      // items are handed out dynamically, longest first: every CTA takes the
      // next item of the cost-sorted list when it is ready for one (greedy
      // longest-processing-time scheduling)
      for (uint32_t r = 0; ok; ++r) {
        const int slot = r & 1;
        if (r >= 2 && !(ok = mbar_wait(&bars[kBarItemEmpty + slot], ((r >> 1) - 1) & 1, wc, 4)))
          break;
        const int got = atomicAdd(prm.work_next, 1);
        const int it = got < n_items ? got : -1;
        s_item[slot] = it;
        mbar_arrive(&bars[kBarItemFull + slot]);
        if (it < 0) break;
        const Item w = prm.items[it];
        const int n_tiles = (w.e_end - w.e_begin + C::EPT - 1) / C::EPT;
        if (n_tiles == 0) continue;
        if (q_uses > 0 && !(ok = mbar_wait(&bars[kBarQEmpty], (q_uses - 1) & 1, wc, 1))) break;
        mbar_arrive_expect_tx(&bars[kBarQFull], w.nh * C::kQTileBytes);
        for (int t = 0; t < w.nh; ++t)
          for (int cb = 0; cb < C::KB; ++cb)
            tma_load_3d(sQ + t * C::kQTileBytes + cb * C::kBlockBytes, &tm_q, &bars[kBarQFull],
                        cb * 64, w.qh0 + t, w.q_row0 + w.row_begin);
        ++q_uses;
        auto tile_rows = [&](int jt, int32_t (&rows)[C::EPT]) {
#pragma unroll
          for (int e = 0; e < C::EPT; ++e) {
            const int idx = w.e_begin + jt * C::EPT + e;
            rows[e] = oob_row;
            if (idx < w.e_end) {
              const int32_t pg = prm.entries[idx].phys_page;
              if (pg >= 0 && pg < prm.n_pages) rows[e] = pg * P;
              else atomicOr(prm.error_word, static_cast<int>(RK_DEV_BAD_PAGE));
            }
          }
        };
        // K runs one tile ahead of V: with two V stages a V load waits for
        // an older PV to finish, and K loads queued behind it arrived late
        for (int j = -1; j < n_tiles; ++j) {
          int32_t rows[C::EPT];
          if (j + 1 < n_tiles) {
            tile_rows(j + 1, rows);
            const int st = k_issued % SK;
            const uint32_t u = k_issued / SK;
            if (u > 0 && !(ok = mbar_wait(&k_empty[st], (u - 1) & 1, wc, 2))) break;
            mbar_arrive_expect_tx(&k_full[st], C::kKVTileBytes);
#pragma unroll
            for (int e = 0; e < C::EPT; ++e)
#pragma unroll
              for (int cb = 0; cb < C::KB; ++cb)
                tma_load_2d(sK + st * C::kKVTileBytes + cb * C::kBlockBytes + e * P * 128, &tm_k,
                            &k_full[st], cb * 64, rows[e]);
            ++k_issued;
          }
          if (j >= 0) {
            tile_rows(j, rows);
            const int st = v_issued % SV;
            const uint32_t u = v_issued / SV;
            if (u > 0 && !(ok = mbar_wait(&v_empty[st], (u - 1) & 1, wc, 3))) break;
            mbar_arrive_expect_tx(&v_full[st], C::kKVTileBytes);
#pragma unroll
            for (int e = 0; e < C::EPT; ++e)
#pragma unroll
              for (int cb = 0; cb < C::KB; ++cb)
                tma_load_2d(sV + st * C::kKVTileBytes + cb * C::kBlockBytes + e * P * 128, &tm_v,
                            &v_full[st], cb * 64, rows[e]);
            ++v_issued;
          }
        }
      }
      if (!ok) {
        // drain: let every copy this thread started land before the CTA exits
        for (uint32_t k = (k_issued > SK ? k_issued - SK : 0); k < k_issued; ++k)
          mbar_wait_drain(&k_full[k % SK], (k / SK) & 1);
        for (uint32_t k = (v_issued > SV ? v_issued - SV : 0); k < v_issued; ++k)
          mbar_wait_drain(&v_full[k % SV], (k / SV) & 1);
        if (q_uses > 0) mbar_wait_drain(&bars[kBarQFull], (q_uses - 1) & 1);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------- MMA issuers
    // One issuing thread per Q tile (warp 1: tile 0, warp 3: tile 1): a
    // tcgen05.mma holds its issuing thread until the tensor pipe takes it,
    // so each tile's MMAs need their own thread.  Per KV tile j, issuer t
    // puts S_t(j + 1) into the shared S buffer, then issues PV_t(j) once P_t(j)
    // is stored.  The S buffer is taken in a fixed global order
    // (S_0(j), S_1(j), S_0(j + 1), ...): S number n waits until the softmax
    // has read S number n - 1 (kBarSFree completes once per S), so the next S
    // of one tile is computed while the other tile runs its exponentials.
    // K / V stages, Q buffers and the Q-rotation handoff are released by both
    // issuers (counts of 2); an issuer whose tile is absent from an item (a
    // single q head) still steps through them.
    if (lane == 0) {
      const int t = warp == 1 ? 0 : 1;
      constexpr uint32_t idesc_s = idesc_bf16_f32(kRowsPerTile, kKeysPerTile, false);
      constexpr uint32_t idesc_o = idesc_bf16_f32(kRowsPerTile, D, true);
      const uint32_t sQa = smem_u32(sQ) + t * C::kQTileBytes, sKa = smem_u32(sK), sVa = smem_u32(sV);
      const uint32_t tO = tmem + C::col_o(t), tP = tmem + C::col_p(t);
      uint64_t* k_avail = fuse ? k_ready : k_full;
      uint32_t kv_iter = 0, q_uses = 0, qrd_uses = 0, p_phase = 0, o_uses = 0;
      uint32_t sf_uses = 0;  // phases of this issuer's kBarSFree consumed
      bool any_s = false;    // this issuer has put an S in the buffer before
      bool ok = true;
      // S_t = Q_t K^T (M=128, N=128, K=D) into the shared S buffer.  The
      // softmax that reads the S before it in the global order arrives on
      // this issuer's kBarSFree, so each issuer waits every phase of its own
      // barrier in order (a parity wait that skipped phases could match an
      // older completed phase of the same parity).  The kernel's very first S
      // (tile 0's) has no predecessor.
      auto issue_s = [&](int kst) {
        if (t == 1 || any_s) {
          if (!(ok = mbar_wait(&bars[kBarSFree + t], sf_uses & 1, wc, 18))) return;
          ++sf_uses;
        }
        any_s = true;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * C::kBlockBytes + (kk & 3) * 32;
          const uint64_t a = desc_sw128(sQa + off, 16, 1024);
          const uint64_t bd = desc_sw128(sKa + kst * C::kKVTileBytes + off, 16, 1024);
          mma_bf16_ss(tmem + C::kColS, a, bd, idesc_s, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bars[kBarSFull + t]);
      };
      // O_t (+)= P_t V (M=128, N=D, K=128), P_t read from TMEM
      auto issue_pv = [&](int vst, bool acc) {
#pragma unroll
        for (int kk = 0; kk < kKeysPerTile / 16; ++kk) {
          const uint64_t bd =
              desc_sw128(sVa + vst * C::kKVTileBytes + kk * 16 * 128, C::kBlockBytes, 1024);
          mma_bf16_ts(tO, tP + kk * 8, bd, idesc_o, (acc || kk > 0) ? 1u : 0u);
        }
        tc_commit(&bars[kBarPVDone + t]);
      };
      for (uint32_t r = 0; ok; ++r) {
        const int it = next_item(bars, s_item, r, wc, 5, ok);
        if (it < 0) break;
        const Item w = prm.items[it];
        const int n_tiles = (w.e_end - w.e_begin + C::EPT - 1) / C::EPT;
        if (n_tiles == 0) continue;
        const int nh = w.nh;
        const bool active = t < nh;
        if (fuse) {
          if (!(ok = mbar_wait(&bars[kBarQReady], qrd_uses & 1, wc, 10))) break;
          ++qrd_uses;
        } else if (!(ok = mbar_wait(&bars[kBarQFull], q_uses & 1, wc, 10))) {
          break;
        }
        ++q_uses;
        int dcur = fuse ? __ldg(&prm.entries[w.e_begin].delta) : 0;
        // K stage of KV tile jn, resident (and, fused, Q rotated for it)
        auto k_tile = [&](int jn) -> int {
          if (fuse && jn > 0) {
            const int dn = __ldg(&prm.entries[w.e_begin + jn * C::EPT].delta);
            if (dn != dcur) {
              // every S that read the old rotation precedes this commit
              tc_commit(&bars[kBarQFree]);
              if (!(ok = mbar_wait(&bars[kBarQReady], qrd_uses & 1, wc, 17))) return 0;
              ++qrd_uses;
              dcur = dn;
            }
          }
          const uint32_t kj = kv_iter + jn;
          const int kst = kj % SK;
          ok = mbar_wait(&k_avail[kst], (kj / SK) & 1, wc, 11);
          return kst;
        };
        {
          const int kst = k_tile(0);
          if (ok && active) issue_s(kst);
          if (ok) tc_commit(&k_empty[kst]);
        }
        for (int j = 0; j < n_tiles && ok; ++j) {
          const uint32_t kj = kv_iter + j;
          const int vst = kj % SV;
          const bool more = j + 1 < n_tiles;
          int kstn = 0;
          if (more) {
            kstn = k_tile(j + 1);
            if (!ok) break;
            if (active) {
              issue_s(kstn);
              if (!ok) break;
            }
          }
          if (!(ok = mbar_wait(&v_full[vst], (kj / SV) & 1, wc, 14))) break;
          if (active) {
            if (!(ok = mbar_wait(&bars[kBarP + t], p_phase, wc, 12))) break;
            p_phase ^= 1;
            if (j == 0 && o_uses > 0 &&
                !(ok = mbar_wait(&bars[kBarOEmpty + t], (o_uses - 1) & 1, wc, 13)))
              break;
            tc_fence_after();
            issue_pv(vst, j > 0);
          }
          if (more) tc_commit(&k_empty[kstn]);
          tc_commit(&v_empty[vst]);
        }
        if (!ok) break;
        if (active) {
          tc_commit(&bars[kBarOFull + t]);
          ++o_uses;
        }
        tc_commit(&bars[kBarQEmpty]);
        kv_iter += n_tiles;
      }
      // make sure no MMA still writes TMEM when it is released
      tc_commit(&bars[kBarDrain + t]);
      mbar_wait_drain(&bars[kBarDrain + t], 0);
    }
  } else if (warp == 2) {
    // ------------------------------------------- RoPE relocation (fused)
    // q . R(d) k = (R(-d) q) . k: the Q tiles are rotated by -d once per run
    // of tiles whose keys share the relocation d (a cached segment), so the
    // K tiles go to the tensor cores as loaded.  A tile whose pages carry
    // different deltas (a segment boundary inside the tile) has those pages
    // rotated by their delta minus the Q rotation's.  Before each new Q
    // rotation the original Q is fetched again, so every Q element is rounded
    // to bf16 once.
    if (fuse) {
      const int rt = lane;
      const int c = rt % (D / 16);
      uint32_t k_seen = 0, q_uses = 0, qf_uses = 0, qr_uses = 0;
      int tab_delta = 0;
      uint64_t cos2[4], sin2[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        cos2[k] = f2_pack(1.f, 1.f);
        sin2[k] = f2_pack(0.f, 0.f);
      }
      auto table = [&](int delta) {
        if (delta != tab_delta) {
          rope_table(delta, c, prm.inv_freq, cos2, sin2);
          tab_delta = delta;
        }
      };
      bool ok = true;
      for (uint32_t r = 0; ok; ++r) {
        const int it = next_item(bars, s_item, r, wc, 5, ok);
        if (it < 0) break;
        const Item w = prm.items[it];
        const int n_tiles = (w.e_end - w.e_begin + C::EPT - 1) / C::EPT;
        if (n_tiles == 0) continue;
        if (!(ok = mbar_wait(&bars[kBarQFull], q_uses & 1, wc, 31))) break;
        ++q_uses;
        int dq = prm.entries[w.e_begin].delta;
        if (dq != 0) {
          table(-dq);
          for (int t = 0; t < w.nh; ++t)
            rope_rotate_rows<D>(sQ + t * C::kQTileBytes, 0, kRowsPerTile, rt, cos2, sin2);
        }
        fence_proxy_async_smem();
        mbar_arrive(&bars[kBarQReady]);
        for (int j = 0; j < n_tiles && ok; ++j, ++k_seen) {
          const int dt = prm.entries[w.e_begin + j * C::EPT].delta;
          if (j > 0 && dt != dq) {
            if (!(ok = mbar_wait(&bars[kBarQFree], qf_uses & 1, wc, 32))) break;
            ++qf_uses;
            if (rt == 0) {
              mbar_arrive_expect_tx(&bars[kBarQReload], w.nh * C::kQTileBytes);
              for (int t = 0; t < w.nh; ++t)
                for (int cb = 0; cb < C::KB; ++cb)
                  tma_load_3d(sQ + t * C::kQTileBytes + cb * C::kBlockBytes, &tm_q,
                              &bars[kBarQReload], cb * 64, w.qh0 + t, w.q_row0 + w.row_begin);
            }
            if (!(ok = mbar_wait(&bars[kBarQReload], qr_uses & 1, wc, 33))) {
              // let the copy this warp started land before the CTA exits
              if (rt == 0) mbar_wait_drain(&bars[kBarQReload], qr_uses & 1);
              break;
            }
            ++qr_uses;
            if (dt != 0) {
              table(-dt);
              for (int t = 0; t < w.nh; ++t)
                rope_rotate_rows<D>(sQ + t * C::kQTileBytes, 0, kRowsPerTile, rt, cos2, sin2);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars[kBarQReady]);
            dq = dt;
          }
          const int st = k_seen % SK;
          if (!(ok = mbar_wait(&k_full[st], (k_seen / SK) & 1, wc, 30))) break;
          uint8_t* tile = sK + st * C::kKVTileBytes;
          for (int e = 1; e < C::EPT; ++e) {
            const int idx = w.e_begin + j * C::EPT + e;
            if (idx >= w.e_end) break;
            const int de = prm.entries[idx].delta;
            if (de == dq) continue;
            table(de - dq);
            rope_rotate_rows<D>(tile, e * P, e * P + P, rt, cos2, sin2);
          }
          fence_proxy_async_smem();
          mbar_arrive(&k_ready[st]);
        }
      }
    }
  }
  } else {
    // ------------------------------------------------------------ softmax
    setmaxnreg_inc<kRegsSoftmax>();
    const int t = (warp - 4) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_base + C::kColS;
    const uint32_t tP = tmem + lane_base + C::col_p(t);
    const uint32_t tO = tmem + lane_base + C::col_o(t);
    const float sl2 = prm.scale_log2;
    const int T = prm.total_tokens;
    uint32_t s_phase = 0, o_uses = 0;
    uint32_t n_pv = 0;  // PVs of this Q tile issued before the current tile
    bool ok = true;
    for (uint32_t r = 0; ok; ++r) {
      const int it = next_item(bars, s_item, r, wc, 6, ok);
      if (it < 0) break;
      const Item w = prm.items[it];
      if (t >= w.nh) continue;
      const int n_tiles = (w.e_end - w.e_begin + C::EPT - 1) / C::EPT;
      const int i = w.row_begin + row;
      const bool valid = i < w.row_end;
      const int h = w.qh0 + t;
      const int64_t orow = static_cast<int64_t>(w.q_row0 + i) * prm.hq + h;
      const int64_t lse_idx =
          (static_cast<int64_t>(w.layer) * prm.hq + h) * T + (w.q_row0 - w.layer * T) + i;
      if (n_tiles == 0) {
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(prm.o + orow * D);
          for (int k = 0; k < D / 8; ++k) dst[k] = make_uint4(0, 0, 0, 0);
          if (prm.lse) prm.lse[lse_idx] = -INFINITY;
        }
        continue;
      }
      const int window = w.window;
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < n_tiles && ok; ++j) {
        // pages of this tile (loaded before the wait, so their latency hides)
        int lp[C::EPT], nv[C::EPT];
#pragma unroll
        for (int e = 0; e < C::EPT; ++e) {
          const int idx = w.e_begin + j * C::EPT + e;
          if (idx < w.e_end) {
            const int4 en = *reinterpret_cast<const int4*>(prm.entries + idx);
            lp[e] = en.y;
            nv[e] = en.w;
          } else {
            lp[e] = 0;
            nv[e] = 0;
          }
        }
        if (!(ok = mbar_wait(&bars[kBarSFull + t], s_phase, wc, 20))) break;
        s_phase ^= 1;
        tc_fence_after();
        float s[kKeysPerTile];
        tmem_ld_x128_wait(tS, s);
        // S is in registers: the issuer of the next S in the global order
        // (S_1 of this tile after S_0 of a two-head item, else an S_0) may
        // put it in the buffer
        tc_fence_before();
        mbar_arrive(&bars[kBarSFree + ((t == 0 && w.nh == 2) ? 1 : 0)]);
        bool full = true;
#pragma unroll
        for (int e = 0; e < C::EPT; ++e) full = full && nv[e] == P;
        full = full && lp[C::EPT - 1] + P - 1 <= i && (window < 0 || lp[0] > i - window);
        if (!full) {
#pragma unroll
          for (int cc = 0; cc < kKeysPerTile; ++cc) {
            const int e = cc / P, rr = cc % P;
            const int jpos = lp[e] + rr;
            const bool vis = rr < nv[e] && jpos <= i && (window < 0 || jpos > i - window);
            s[cc] = vis ? s[cc] : -INFINITY;
          }
        }
        // row max: 3-input max over 8 independent chains, then a tree
        float mx8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx8[k] = fmax3(s[k], s[8 + k], s[16 + k]);
#pragma unroll
        for (int cc = 24; cc < kKeysPerTile; cc += 16)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx8[k] = fmax3(mx8[k], s[cc + k], s[cc + 8 + k]);
        const float mx = fmaxf(fmax3(mx8[0], mx8[1], mx8[2]),
                               fmax3(fmax3(mx8[3], mx8[4], mx8[5]), mx8[6], mx8[7]));
        const float m_new = fmaxf(m_ref, mx * sl2);
        const bool resc = m_new > m_ref + kRescaleLog2;
        if (j > 0 && __any_sync(0xffffffffu, resc)) {
          // O holds the sum through the previous tile's PV: let it finish
          if (!(ok = mbar_wait(&bars[kBarPVDone + t], (n_pv - 1) & 1, wc, 23))) break;
          tc_fence_after();
          const float alpha = resc ? ex2_approx(m_ref - m_new) : 1.f;
#pragma unroll
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t v[32];
            tmem_ld_x32(tO + 32 * cc, v);
            tmem_ld_wait(v);
#pragma unroll
            for (int k = 0; k < 32; ++k) v[k] = __float_as_uint(__uint_as_float(v[k]) * alpha);
            tmem_st_x32(tO + 32 * cc, v);
          }
          tmem_st_wait();
          if (resc) l *= alpha;
        }
        if (resc) m_ref = m_new;
        const float m_use = m_ref == -INFINITY ? 0.f : m_ref;
        const uint64_t scale2 = f2_pack(sl2, sl2);
        const uint64_t neg_m2 = f2_pack(-m_use, -m_use);
        uint64_t acc2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          float* sh = s + 64 * half;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const uint64_t x2 = f2_fma(f2_pack(sh[2 * k], sh[2 * k + 1]), scale2, neg_m2);
            f2_unpack(x2, sh[2 * k], sh[2 * k + 1]);
          }
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            sh[2 * k] = ex2_approx(sh[2 * k]);
            sh[2 * k + 1] = ex2_approx(sh[2 * k + 1]);
          }
#pragma unroll
          for (int k = 0; k < 32; ++k)
            acc2[k & 1] = f2_add(acc2[k & 1], f2_pack(sh[2 * k], sh[2 * k + 1]));
        }
        // P_t still feeds the previous PV until that completes: waited only
        // now, so the exponentials overlap that PV (every phase of the
        // barrier is waited, across items too, so none is skipped)
        if (n_pv > 0) {
          if (!(ok = mbar_wait(&bars[kBarPVDone + t], (n_pv - 1) & 1, wc, 24))) break;
          tc_fence_after();
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const float* sh = s + 64 * half;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t pk[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
              const int kk = 16 * q + k;
              pk[k] = pack_bf16x2(sh[2 * kk], sh[2 * kk + 1]);
            }
            tmem_st_x16(tP + 32 * half + 16 * q, pk);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars[kBarP + t]);
        ++n_pv;
        float a0, a1, b0, b1;
        f2_unpack(acc2[0], a0, a1);
        f2_unpack(acc2[1], b0, b1);
        l += (a0 + a1) + (b0 + b1);
      }
      if (!ok) break;
      // epilogue: O / l -> bf16
      if (!(ok = mbar_wait(&bars[kBarOFull + t], o_uses & 1, wc, 21))) break;
      ++o_uses;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t v[32];
        tmem_ld_x32(tO + 32 * cc, v);
        tmem_ld_wait(v);
        if (valid) {
          uint32_t pk[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            pk[k] = pack_bf16x2(__uint_as_float(v[2 * k]) * inv, __uint_as_float(v[2 * k + 1]) * inv);
          uint4* dst = reinterpret_cast<uint4*>(prm.o + orow * D + 32 * cc);
#pragma unroll
          for (int k = 0; k < 4; ++k)
            dst[k] = make_uint4(pk[4 * k], pk[4 * k + 1], pk[4 * k + 2], pk[4 * k + 3]);
        }
      }
      if (valid && prm.lse)
        prm.lse[lse_idx] = l > 0.f ? (m_ref + __log2f(l)) * 0.6931471805599453f : -INFINITY;
      tc_fence_before();
      mbar_arrive(&bars[kBarOEmpty + t]);
    }
  }

  tc_fence_before();
  __syncthreads();
  // the last CTA to finish leaves the work counter at 0 for the next launch
  if (threadIdx.x == 0 && atomicAdd(prm.work_done, 1) == static_cast<int>(gridDim.x) - 1) {
    *prm.work_next = 0;
    *prm.work_done = 0;
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode_fn() {
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

template <int D, int P>
static cudaError_t launch_typed(const PrefillLaunchArgs& a, cudaStream_t stream) {
  using C = PrefillCfg<D, P>;
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return cudaErrorNotSupported;
  CUtensorMap tq, tk, tv;
  {
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(a.hq),
                                static_cast<cuuint64_t>(a.n_layers) * a.total_tokens};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(a.hq) * D * 2};
    const cuuint32_t box[3] = {64, 1, kRowsPerTile};
    const cuuint32_t es[3] = {1, 1, 1};
    if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.q), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const cuuint64_t pdims[2] = {static_cast<cuuint64_t>(D),
                               static_cast<cuuint64_t>(a.n_pages) * P};
  const cuuint64_t pstrides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t pbox[2] = {64, static_cast<cuuint32_t>(P)};
  const cuuint32_t pes[2] = {1, 1};
  if (enc(&tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.k_pool), pdims, pstrides,
          pbox, pes, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (enc(&tv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.v_pool), pdims, pstrides,
          pbox, pes, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(segpaged_prefill_kernel<D, P>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  PrefillParams prm;
  prm.items = a.items;
  prm.n_items = a.n_items;
  prm.work_next = a.work_next;
  prm.work_done = a.work_done;
  prm.error_word = a.error_word;
  prm.timeout_site = a.timeout_site;
  prm.entries = a.entries;
  prm.o = static_cast<__nv_bfloat16*>(a.o);
  prm.lse = a.lse;
  prm.hq = a.hq;
  prm.total_tokens = a.total_tokens;
  prm.n_pages = a.n_pages;
  prm.scale_log2 = a.scale_log2;
  prm.fuse_rope = a.fuse_rope;
  for (int m = 0; m < 64; ++m) prm.inv_freq[m] = m < D / 2 ? pow(a.rope_theta, -2.0 * m / D) : 0.0;
  segpaged_prefill_kernel<D, P><<<sms, kPrefillThreads, C::kSmemBytes, stream>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

cudaError_t launch_prefill_args(const PrefillLaunchArgs& a, cudaStream_t stream) {
  if (a.d == 128 && a.p == 64) return launch_typed<128, 64>(a, stream);
  if (a.d == 128 && a.p == 16) return launch_typed<128, 16>(a, stream);
  if (a.d == 64 && a.p == 64) return launch_typed<64, 64>(a, stream);
  if (a.d == 64 && a.p == 16) return launch_typed<64, 16>(a, stream);
  return cudaErrorInvalidValue;
}

}  // namespace rk

