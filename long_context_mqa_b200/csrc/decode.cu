// Decode step of the full-attention + selection layer (one query token per sequence, the
// query at position t = N-1 of an N-token K/V cache).
//
// Exact head-summed probabilities need each head's logsumexp over the whole row before any
// token's score is final, so the cache is scanned twice:
//
//   pass 1  K only.  S^T = K_tile Q^T on tcgen05 (M = 128 keys in TMEM lanes, N = H heads);
//           each thread owns one key lane and keeps a running (max, sum) per head in
//           registers; one cross-lane merge per work segment -> partial (m, l) per head.
//   combine partial (m, l) -> lse per head.
//   pass 2  K and V.  S^T again; p = exp2(s*c - lse2) exactly (no rescaling); the head sum
//           is an in-thread reduction (score of the thread's key); P^T (bf16) goes to shared
//           memory as an MN-major operand and O^T += V^T P^T accumulates in TMEM. Scores of
//           the older tokens go to a global buffer and a 2048-bin histogram of their top bits.
//   combine partial outputs; radix selection (select.cu) turns histogram + scores into idx.
//
// Work split: the flattened (sequence, 128-key tile) space is cut into G contiguous ranges,
// one per CTA (G = number of SMs); a range may cross a sequence boundary, so a CTA handles
// one or more "segments", each producing one partial record. Pass 2 walks its range in
// reverse order so that the keys pass 1 touched last are re-read first (L2 hits).
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = tcgen05 issuer (and TMEM
// owner), warps 2..5 = the 128 softmax threads (warp w reads TMEM lanes 32*(w%4)..+31).
// Every wait is bounded; on timeout the kernel records it in the status word and unwinds.
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace dec {

constexpr int TILE = 128;
constexpr int NTHREADS = 192;
constexpr int SOFTMAX_BAR = 1;  // named barrier id of the 128 softmax threads

__device__ __forceinline__ void softmax_bar() { asm volatile("bar.sync %0, 128;" ::"n"(SOFTMAX_BAR) : "memory"); }

__device__ __forceinline__ void tile_range(const DecParams& p, int cta, long long& t0, long long& t1) {
  t0 = p.total_tiles * cta / p.G;
  t1 = p.total_tiles * (cta + 1) / p.G;
}

// bounded wait that also gives up when another role already aborted
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, long long limit, volatile int* abort_flag,
                                         DevStatus* st, unsigned where) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const long long t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(a, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit) {
      *abort_flag = 1;
      report_status(st, kStatusTimeout, where);
      return false;
    }
  }
}

// Warp-collective form: lane 0 waits, every lane gets the same answer, so the
// warp-synchronous tcgen05.ld that follows is never reached by only part of the warp.
__device__ __forceinline__ bool warp_wait_bar(uint64_t* bar, uint32_t parity, long long limit,
                                              volatile int* abort_flag, DevStatus* st, unsigned where) {
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(bar, parity, limit, abort_flag, st, where) ? 1 : 0;
  ok = __shfl_sync(0xffffffffu, ok, 0);
  return ok != 0;
}

// ------------------------------------------------------------------------------------------
// pass 1: per-head (max, sum) partials of exp2(s * c)
// ------------------------------------------------------------------------------------------
template <int H, int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    dec_pass1_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, DecParams p) {
  constexpr int KST = 5;
  constexpr int KT_BYTES = TILE * D * 2;
  constexpr int Q_BYTES = H * D * 2;
  constexpr int NKB = D / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                // 2 buffers
  uint8_t* sK = smem + 2 * Q_BYTES;  // KST stages
  __shared__ __align__(8) uint64_t k_full[KST], k_empty[KST], s_full[2], s_empty[2], q_full[2], q_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ float red[4][H][2];

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  long long t0, t1;
  tile_range(p, cta, t0, t1);
  const long long limit = p.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 4);
      mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, 128); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmQ);
      uint32_t j = 0;
      int seg = 0;
      bool ok = true;
      for (long long t = t0; t < t1 && ok; ++seg) {
        const int b = (int)(t / p.tps);
        const long long seg_end = t1 < (long long)(b + 1) * p.tps ? t1 : (long long)(b + 1) * p.tps;
        const int qb = seg & 1;
        if (!wait_bar(&q_empty[qb], ((seg >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 101)) { ok = false; break; }
        mbar_expect_tx(&q_full[qb], Q_BYTES);
        for (int kb = 0; kb < NKB; ++kb) tma_load_3d(sQ + qb * Q_BYTES + kb * (H * 128), &tmQ, &q_full[qb], kb * 64, 0, b);
        for (; t < seg_end; ++t, ++j) {
          const int lt = (int)(t - (long long)b * p.tps);
          const int s = j % KST;
          if (!wait_bar(&k_empty[s], ((j / KST) & 1) ^ 1, limit, &abort_flag, p.st, 102)) { ok = false; break; }
          mbar_expect_tx(&k_full[s], KT_BYTES);
          for (int kb = 0; kb < NKB; ++kb)
            tma_load_3d(sK + s * KT_BYTES + kb * (TILE * 128), &tmK, &k_full[s], kb * 64, lt * TILE, b);
        }
      }
      if (!ok) {  // let the copies already issued land before the CTA exits
        for (uint32_t jj = (j > KST ? j - KST : 0); jj < j; ++jj)
          mbar_wait(&k_full[jj % KST], (jj / KST) & 1, limit);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, H, 0, 0);
      uint32_t j = 0;
      int seg = 0;
      bool ok = true;
      for (long long t = t0; t < t1 && ok; ++seg) {
        const int b = (int)(t / p.tps);
        const long long seg_end = t1 < (long long)(b + 1) * p.tps ? t1 : (long long)(b + 1) * p.tps;
        const int qb = seg & 1;
        if (!wait_bar(&q_full[qb], (seg >> 1) & 1, limit, &abort_flag, p.st, 111)) { ok = false; break; }
        const uint32_t qaddr = smem_u32(sQ + qb * Q_BYTES);
        for (; t < seg_end; ++t, ++j) {
          const int s = j % KST, buf = j & 1;
          if (!wait_bar(&k_full[s], (j / KST) & 1, limit, &abort_flag, p.st, 112)) { ok = false; break; }
          if (!wait_bar(&s_empty[buf], ((j >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 113)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kaddr = smem_u32(sK + s * KT_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sdesc(kaddr + (kk / 4) * (TILE * 128) + (kk % 4) * 32, 16, 1024);
            const uint64_t bq = sdesc(qaddr + (kk / 4) * (H * 128) + (kk % 4) * 32, 16, 1024);
            umma_bf16(tmem + buf * H, a, bq, IDESC, kk > 0);
          }
          umma_commit(&s_full[buf]);
          umma_commit(&k_empty[s]);
        }
        umma_commit(&q_empty[qb]);
      }
    }
  } else {
    // softmax threads: lane quarter of this warp
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int wg_tid = (warp - 2) * 32 + lane;
    const float c = p.c;
    uint32_t j = 0;
    int seg = 0;
    for (long long t = t0; t < t1; ++seg) {
      const int b = (int)(t / p.tps);
      const long long seg_end = t1 < (long long)(b + 1) * p.tps ? t1 : (long long)(b + 1) * p.tps;
      const int slot = cta * p.segmax + (b - (int)(t0 / p.tps));
      float m[H], l[H];
#pragma unroll
      for (int h = 0; h < H; ++h) { m[h] = -1e30f; l[h] = 0.f; }
      bool ok = true;
      for (; t < seg_end; ++t, ++j) {
        const int lt = (int)(t - (long long)b * p.tps);
        const int buf = j & 1;
        if (!warp_wait_bar(&s_full[buf], (j >> 1) & 1, limit, &abort_flag, p.st, 121)) { ok = false; break; }
        tc_fence_after();
        const int key = lt * TILE + row;
        // two halves of 32 columns keep the register footprint below the spill limit
#pragma unroll
        for (int half = 0; half < H / 32; ++half) {
          float v[32];
          tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + buf * H + half * 32, v);
          tmem_ld_wait();
          if (half == H / 32 - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_empty[buf]);
          }
          if (key < p.N) {
#pragma unroll
            for (int x2 = 0; x2 < 32; ++x2) {
              const int h = half * 32 + x2;
              const float x = v[x2] * c;
              const float dl = x - m[h];
              const float e = fast_exp2(-fabsf(dl));
              const bool up = dl > 0.f;
              l[h] = up ? fmaf(l[h], e, 1.f) : l[h] + e;
              m[h] = up ? x : m[h];
            }
          }
        }
      }
      if (!ok) { t = t1; }
      // merge the 128 lanes: warp shuffle, then the 4 warps through shared memory
#pragma unroll
      for (int h = 0; h < H; ++h) {
        float mm = m[h], ll = l[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, mm, off);
          const float l2 = __shfl_xor_sync(0xffffffffu, ll, off);
          const float mx = fmaxf(mm, m2);
          ll = ll * fast_exp2(mm - mx) + l2 * fast_exp2(m2 - mx);
          mm = mx;
        }
        if (lane == 0) { red[warp - 2][h][0] = mm; red[warp - 2][h][1] = ll; }
      }
      softmax_bar();
      if (wg_tid < H) {
        float mm = red[0][wg_tid][0], ll = red[0][wg_tid][1];
        for (int w = 1; w < 4; ++w) {
          const float m2 = red[w][wg_tid][0], l2 = red[w][wg_tid][1];
          const float mx = fmaxf(mm, m2);
          ll = ll * fast_exp2(mm - mx) + l2 * fast_exp2(m2 - mx);
          mm = mx;
        }
        p.ml[(size_t)slot * 2 * H + wg_tid] = mm;
        p.ml[(size_t)slot * 2 * H + H + wg_tid] = ll;
      }
      softmax_bar();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 128); }
}

// ------------------------------------------------------------------------------------------
// combine pass-1 partials -> lse (log2 domain for pass 2, natural log for the caller)
// ------------------------------------------------------------------------------------------
template <int H>
__global__ void dec_lse_combine_kernel(DecParams p) {
  const int b = blockIdx.x, h = threadIdx.x;
  float M = -1e30f, L = 0.f;
  for (int cta = 0; cta < p.G; ++cta) {
    long long t0, t1;
    tile_range(p, cta, t0, t1);
    const long long lo = t0 > (long long)b * p.tps ? t0 : (long long)b * p.tps;
    const long long hi = t1 < (long long)(b + 1) * p.tps ? t1 : (long long)(b + 1) * p.tps;
    if (lo >= hi) continue;
    const int slot = cta * p.segmax + (b - (int)(t0 / p.tps));
    const float m = p.ml[(size_t)slot * 2 * H + h], l = p.ml[(size_t)slot * 2 * H + H + h];
    const float mx = fmaxf(M, m);
    L = L * exp2f(M - mx) + l * exp2f(m - mx);
    M = mx;
  }
  const float lse2 = M + log2f(L);
  p.lse2[b * H + h] = lse2;
  p.lse_out[b * H + h] = lse2 * 0.69314718055994531f;
}

// ------------------------------------------------------------------------------------------
// pass 2: exact probabilities, output partials, head-summed scores, histogram
// ------------------------------------------------------------------------------------------
template <int H, int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    dec_pass2_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, DecParams p) {
  static_assert(H == 64 && D == 128, "decode pass 2 is instantiated for 64 heads x 128");
  constexpr int ST = 2;
  constexpr int KT_BYTES = TILE * D * 2;
  constexpr int Q_BYTES = H * D * 2;
  constexpr int P_BYTES = TILE * H * 2;
  constexpr int NKB = D / 64;
  constexpr int NBINS = 2048;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                           // 2 x Q
  uint8_t* sK = sQ + 2 * Q_BYTES;               // ST x K tile
  uint8_t* sV = sK + ST * KT_BYTES;             // ST x V tile
  uint8_t* sP = sV + ST * KT_BYTES;             // 2 x P^T
  uint32_t* shist = (uint32_t*)(sP + 2 * P_BYTES);
  __shared__ __align__(8) uint64_t k_full[ST], k_empty[ST], v_full[ST], v_empty[ST], s_full[2], s_empty[2], p_full[2],
      p_empty[2], q_full[2], q_empty[2], o_full, o_empty;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ float slse[H];

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  long long t0, t1;
  tile_range(p, cta, t0, t1);
  const long long limit = p.wait_ns;
  const uint32_t tS = 0, tO = 2 * H;  // TMEM column offsets

  for (int i = threadIdx.x; i < NBINS; i += NTHREADS) shist[i] = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4); mbar_init(&p_empty[i], 1);
      mbar_init(&q_full[i], 1); mbar_init(&q_empty[i], 1);
    }
    mbar_init(&o_full, 1); mbar_init(&o_empty, 4);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  // segments are walked from the end of the range backwards, tiles likewise
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV); tma_prefetch_desc(&tmQ);
      uint32_t j = 0;
      int seg = 0;
      bool ok = true;
      for (long long t = t1 - 1; t >= t0 && ok; ++seg) {
        const int b = (int)(t / p.tps);
        const long long seg_lo = t0 > (long long)b * p.tps ? t0 : (long long)b * p.tps;
        const int qb = seg & 1;
        if (!wait_bar(&q_empty[qb], ((seg >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 201)) { ok = false; break; }
        mbar_expect_tx(&q_full[qb], Q_BYTES);
        for (int kb = 0; kb < NKB; ++kb) tma_load_3d(sQ + qb * Q_BYTES + kb * (H * 128), &tmQ, &q_full[qb], kb * 64, 0, b);
        for (; t >= seg_lo; --t, ++j) {
          const int lt = (int)(t - (long long)b * p.tps);
          const int s = j % ST;
          if (!wait_bar(&k_empty[s], ((j / ST) & 1) ^ 1, limit, &abort_flag, p.st, 202)) { ok = false; break; }
          mbar_expect_tx(&k_full[s], KT_BYTES);
          for (int kb = 0; kb < NKB; ++kb)
            tma_load_3d(sK + s * KT_BYTES + kb * (TILE * 128), &tmK, &k_full[s], kb * 64, lt * TILE, b);
          if (!wait_bar(&v_empty[s], ((j / ST) & 1) ^ 1, limit, &abort_flag, p.st, 203)) { ok = false; ++j; break; }
          mbar_expect_tx(&v_full[s], KT_BYTES);
          for (int kb = 0; kb < NKB; ++kb)
            tma_load_3d(sV + s * KT_BYTES + kb * (TILE * 128), &tmV, &v_full[s], kb * 64, lt * TILE, b);
        }
      }
      if (!ok) {
        for (uint32_t jj = (j > ST ? j - ST : 0); jj < j; ++jj) {
          mbar_wait(&k_full[jj % ST], (jj / ST) & 1, limit);
          mbar_wait(&v_full[jj % ST], (jj / ST) & 1, limit);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, H, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16(D, H, 1, 1);
      uint32_t j = 0;
      int seg = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t jj, bool first, int segi) -> bool {
        const int buf = jj & 1, s = jj % ST;
        if (!wait_bar(&p_full[buf], (jj >> 1) & 1, limit, &abort_flag, p.st, 214)) return false;
        if (!wait_bar(&v_full[s], (jj / ST) & 1, limit, &abort_flag, p.st, 215)) return false;
        if (first && !wait_bar(&o_empty, (segi & 1) ^ 1, limit, &abort_flag, p.st, 216)) return false;
        tc_fence_after();
        const uint32_t vaddr = smem_u32(sV + s * KT_BYTES), paddr = smem_u32(sP + buf * P_BYTES);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          const uint64_t a = sdesc(vaddr + kk * 2048, TILE * 128, 1024);
          const uint64_t bb = sdesc(paddr + kk * 2048, TILE * 128, 1024);
          umma_bf16(tmem + tO, a, bb, IDESC_O, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&p_empty[buf]);
        umma_commit(&v_empty[s]);
        return true;
      };
      for (long long t = t1 - 1; t >= t0 && ok; ++seg) {
        const int b = (int)(t / p.tps);
        const long long seg_lo = t0 > (long long)b * p.tps ? t0 : (long long)b * p.tps;
        const int qb = seg & 1;
        if (!wait_bar(&q_full[qb], (seg >> 1) & 1, limit, &abort_flag, p.st, 211)) { ok = false; break; }
        const uint32_t qaddr = smem_u32(sQ + qb * Q_BYTES);
        int n_in_seg = 0;
        for (; t >= seg_lo; --t, ++j, ++n_in_seg) {
          const int s = j % ST, buf = j & 1;
          if (!wait_bar(&k_full[s], (j / ST) & 1, limit, &abort_flag, p.st, 212)) { ok = false; break; }
          if (!wait_bar(&s_empty[buf], ((j >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 213)) { ok = false; break; }
          tc_fence_after();
          const uint32_t kaddr = smem_u32(sK + s * KT_BYTES);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sdesc(kaddr + (kk / 4) * (TILE * 128) + (kk % 4) * 32, 16, 1024);
            const uint64_t bq = sdesc(qaddr + (kk / 4) * (H * 128) + (kk % 4) * 32, 16, 1024);
            umma_bf16(tmem + tS + buf * H, a, bq, IDESC_S, kk > 0);
          }
          umma_commit(&s_full[buf]);
          umma_commit(&k_empty[s]);
          if (n_in_seg > 0 && !issue_pv(j - 1, n_in_seg == 1, seg)) { ok = false; break; }
        }
        if (!ok) break;
        umma_commit(&q_empty[qb]);
        if (!issue_pv(j - 1, n_in_seg == 1, seg)) { ok = false; break; }
        umma_commit(&o_full);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // key within the tile == TMEM lane == P^T row
    const int wg_tid = (warp - 2) * 32 + lane;
    const float c = p.c;
    const int ncand = p.N - p.W > 0 ? p.N - p.W : 0;
    uint32_t j = 0;
    int seg = 0;
    bool ok = true;
    for (long long t = t1 - 1; t >= t0 && ok; ++seg) {
      const int b = (int)(t / p.tps);
      const long long seg_lo = t0 > (long long)b * p.tps ? t0 : (long long)b * p.tps;
      const int slot = cta * p.segmax + (b - (int)(t0 / p.tps));
      if (wg_tid < H) slse[wg_tid] = p.lse2[b * H + wg_tid];
      softmax_bar();
      for (; t >= seg_lo; --t, ++j) {
        const int lt = (int)(t - (long long)b * p.tps);
        const int buf = j & 1;
        if (!warp_wait_bar(&s_full[buf], (j >> 1) & 1, limit, &abort_flag, p.st, 221)) { ok = false; break; }
        tc_fence_after();
        float v[H];
#pragma unroll
        for (int cc = 0; cc < H / 16; ++cc) {
          float tmp[16];
          tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + tS + buf * H + cc * 16, tmp);
#pragma unroll
          for (int x = 0; x < 16; ++x) v[cc * 16 + x] = tmp[x];
        }
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[buf]);
        const int key = lt * TILE + row;
        const bool valid = key < p.N;
        float score = 0.f;
        uint32_t pk[H / 2];
#pragma unroll
        for (int h = 0; h < H; h += 2) {
          const float p0 = valid ? fast_exp2(fmaf(v[h], c, -slse[h])) : 0.f;
          const float p1 = valid ? fast_exp2(fmaf(v[h + 1], c, -slse[h + 1])) : 0.f;
          score += p0;
          score += p1;
          pk[h / 2] = pack_bf16x2(p0, p1);
        }
        if (!warp_wait_bar(&p_empty[buf], ((j >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 222)) { ok = false; break; }
        const uint32_t prow = smem_u32(sP + buf * P_BYTES);
#pragma unroll
        for (int ch = 0; ch < H / 8; ++ch)
          st_shared_v4(prow + sw128_off(row, ch), pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[buf]);
        if (valid && key < ncand) {
          p.sc[(size_t)b * ncand + key] = score;
          atomicAdd(&shist[__float_as_uint(score) >> 20], 1u);
        }
      }
      if (!ok) break;
      // segment done: fetch O^T (lane = output column d, one TMEM column per head)
      if (!warp_wait_bar(&o_full, seg & 1, limit, &abort_flag, p.st, 223)) { ok = false; break; }
      tc_fence_after();
      float o[H];
#pragma unroll
      for (int cc = 0; cc < H / 16; ++cc) {
        float tmp[16];
        tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + tO + cc * 16, tmp);
#pragma unroll
        for (int x = 0; x < 16; ++x) o[cc * 16 + x] = tmp[x];
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_empty);
      float* dst = p.opart + (size_t)slot * H * D;
#pragma unroll
      for (int h = 0; h < H; ++h) dst[h * D + row] = o[h];
      // flush this sequence's histogram
      softmax_bar();
      for (int i = wg_tid; i < NBINS; i += 128) {
        const uint32_t cnt = shist[i];
        if (cnt) { atomicAdd(&p.hist[(size_t)b * NBINS + i], cnt); shist[i] = 0; }
      }
      softmax_bar();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 256); }
}

// ------------------------------------------------------------------------------------------
// combine output partials (already normalised by the global lse) -> bf16 out
// ------------------------------------------------------------------------------------------
template <int H, int D>
__global__ void dec_out_combine_kernel(DecParams p, __nv_bfloat16* out) {
  const int b = blockIdx.x, h = blockIdx.y, d = threadIdx.x;
  float acc = 0.f;
  for (int cta = 0; cta < p.G; ++cta) {
    long long t0, t1;
    tile_range(p, cta, t0, t1);
    const long long lo = t0 > (long long)b * p.tps ? t0 : (long long)b * p.tps;
    const long long hi = t1 < (long long)(b + 1) * p.tps ? t1 : (long long)(b + 1) * p.tps;
    if (lo >= hi) continue;
    const int slot = cta * p.segmax + (b - (int)(t0 / p.tps));
    acc += p.opart[((size_t)slot * H + h) * D + d];
  }
  out[((size_t)b * H + h) * D + d] = __float2bfloat16_rn(acc);
}

// ------------------------------------------------------------------------------------------
// host launcher
// ------------------------------------------------------------------------------------------
size_t pass1_smem_bytes(int H, int D) { return 1024 + 2 * (size_t)H * D * 2 + 5 * (size_t)TILE * D * 2; }
size_t pass2_smem_bytes(int H, int D) {
  return 1024 + 2 * (size_t)H * D * 2 + 4 * (size_t)TILE * D * 2 + 2 * (size_t)TILE * H * 2 + 2048 * 4;
}

cudaError_t launch_decode_attn(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                               const DecParams& p, __nv_bfloat16* out, cudaStream_t stream) {
  constexpr int H = 64, D = 128;
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(dec_pass1_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)pass1_smem_bytes(H, D));
    cudaFuncSetAttribute(dec_pass2_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)pass2_smem_bytes(H, D));
    configured = true;
  }
  {
    LaunchScope ls("dec_pass1", stream);
    dec_pass1_kernel<H, D><<<p.G, NTHREADS, pass1_smem_bytes(H, D), stream>>>(tmK, tmQ, p);
  }
  {
    LaunchScope ls("dec_lse_combine", stream);
    dec_lse_combine_kernel<H><<<p.B, H, 0, stream>>>(p);
  }
  {
    LaunchScope ls("dec_pass2", stream);
    dec_pass2_kernel<H, D><<<p.G, NTHREADS, pass2_smem_bytes(H, D), stream>>>(tmK, tmV, tmQ, p);
  }
  {
    LaunchScope ls("dec_out_combine", stream);
    dec_out_combine_kernel<H, D><<<dim3(p.B, H), D, 0, stream>>>(p, out);
  }
  return cudaGetLastError();
}

}  // namespace dec
}  // namespace hs2
