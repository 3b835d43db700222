// Decode step of the full-attention + selection layer (one query token per sequence, the
// query at position t = N-1 of an N-token K/V cache).
//
// Exact head-summed probabilities need each head's logsumexp over the whole row before any
// token's score is final, so the cache is scanned twice:
//
//   pass 1  K only.  S^T = K_tile Q^T on tcgen05 (M = 128 keys in TMEM lanes, N = 64 heads).
//           Two softmax warpgroups split the heads (32 each); every thread owns one key lane
//           and keeps, per head, a reference r and a sum l of exp2(s*c - r). r is only moved
//           (with the usual rescale of l) when a value exceeds it by more than 2^64, so the
//           common step is one FFMA, one MUFU ex2, one FADD and one FMNMX per element. One
//           cross-lane merge per work segment -> partial (m, l) per head. CTA 0 also clears the
//           selection histogram for pass 2.
//   pass 2  K and V.  Prologue: the segment's per-head lse from all pass-1 partials of that
//           sequence (the CTA owning the sequence's first tile also writes the caller's lse).
//           S^T again; p = exp2(s*c - lse2) exactly (no rescaling); the head sum is an in-thread
//           reduction (the score of the thread's key); P^T (bf16) goes to shared memory as an
//           MN-major operand and O^T += V^T P^T accumulates in TMEM. Two softmax warpgroups take
//           alternate tiles. Scores of older tokens go to a global buffer and a 2048-bin
//           histogram of their top bits (warp-aggregated shared atomics).
//           The last CTA to finish a sequence scans that sequence's histogram for the bin of
//           its k-th largest score.
//   finish  (select.cu) sum of the output partials -> bf16 out; collect / final selection.
//
// Work split: the flattened (sequence, 128-key tile) space is cut into G contiguous ranges,
// one per CTA (G = number of SMs); a range may cross a sequence boundary, so a CTA handles
// one or more "segments", each producing one partial record. Pass 2 walks its range in
// reverse order so the keys pass 1 touched last are re-read first (L2 hits).
//
// Warp roles: warp 0 = K (and Q) TMA producer, warp 1 = tcgen05 issuer and TMEM owner,
// warp 2 = V producer (pass 2), warps 4..7 and 8..11 = the two softmax warpgroups (warp w
// reads TMEM lanes 32*(w%4)..+31). Every wait is bounded; on timeout the kernel records it
// in the status word and unwinds.
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace dec {

constexpr int TILE = 128;
constexpr int NTHREADS = 384;
constexpr int SM_WG0 = 4;     // first warp of softmax warpgroup 0
constexpr float REF_SLACK = 64.f;

__device__ __forceinline__ void tile_range(const DecParams& p, int cta, long long& t0, long long& t1) {
  t0 = p.total_tiles * cta / p.G;
  t1 = p.total_tiles * (cta + 1) / p.G;
}
// CTA whose range holds flattened tile x
__device__ __forceinline__ int cta_of_tile(const DecParams& p, long long x) {
  return (int)(((x + 1) * p.G - 1) / p.total_tiles);
}
__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

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
// pass 1: per-head (reference, sum) partials of exp2(s * c)
// ------------------------------------------------------------------------------------------
template <int H, int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    dec_pass1_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmQ, DecParams p) {
  constexpr int KST = 5;
  constexpr int KT_BYTES = TILE * D * 2;
  constexpr int Q_BYTES = H * D * 2;
  constexpr int NKB = D / 64;
  constexpr int HW = H / 2;  // heads per warpgroup
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                // 2 buffers
  uint8_t* sK = smem + 2 * Q_BYTES;  // KST stages
  __shared__ __align__(8) uint64_t k_full[KST], k_empty[KST], s_full[2], s_empty[2], q_full[2], q_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ float red[2][4][HW][2];

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  long long t0, t1;
  tile_range(p, cta, t0, t1);
  const long long limit = p.wait_ns;

  if (cta == 0) {  // pass 2 accumulates into the selection histogram and per-sequence counters
    for (int i = threadIdx.x; i < p.B * 2048; i += NTHREADS) p.hist[i] = 0u;
    for (int i = threadIdx.x; i < p.B; i += NTHREADS) p.seq_done[i] = 0;
  }
  {  // the selection bitmap, cleared by all CTAs (the collect kernel sets bits)
    const long long total = (long long)p.B * p.words;
    const long long per = (total + p.G - 1) / p.G;
    const long long w0 = per * cta, w1 = w0 + per < total ? w0 + per : total;
    for (long long i = w0 + threadIdx.x; i < w1; i += NTHREADS) p.bitmap[i] = 0u;
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 8);
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
  griddep_launch_dependents();  // pass 2 may start streaming K/V into freed SMs

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmQ);
      const uint64_t pol = policy_evict_last();  // pass 2 re-reads K: keep it in L2 if possible
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
            tma_load_3d_hint(sK + s * KT_BYTES + kb * (TILE * 128), &tmK, &k_full[s], kb * 64, lt * TILE, b, pol);
        }
      }
      if (!ok)  // let the copies already issued land before the CTA exits
        for (uint32_t jj = (j > KST ? j - KST : 0); jj < j; ++jj) mbar_wait(&k_full[jj % KST], (jj / KST) & 1, limit);
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
  } else if (warp >= SM_WG0) {
    const int wg = (warp - SM_WG0) / 4;  // heads [wg*HW, wg*HW + HW)
    const int wq = (warp - SM_WG0) % 4;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int wg_tid = wq * 32 + lane;
    const float c = p.c;
    uint32_t j = 0;
    for (long long t = t0; t < t1;) {
      const int b = (int)(t / p.tps);
      const long long seg_end = t1 < (long long)(b + 1) * p.tps ? t1 : (long long)(b + 1) * p.tps;
      const int slot = cta * p.segmax + (b - (int)(t0 / p.tps));
      const long long seg_first = t;
      float r[HW], l[HW];
#pragma unroll
      for (int h = 0; h < HW; ++h) { r[h] = -INFINITY; l[h] = 0.f; }
      // after a failed wait every later wait returns at once: keep the loop and barrier
      // structure identical across warps, skip only the work
      bool ok = !abort_flag;
      for (; t < seg_end; ++t, ++j) {
        const int lt = (int)(t - (long long)b * p.tps);
        const int buf = j & 1;
        if (!ok) continue;
        if (!warp_wait_bar(&s_full[buf], (j >> 1) & 1, limit, &abort_flag, p.st, 121)) { ok = false; continue; }
        tc_fence_after();
        float v[HW];
        tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + buf * H + wg * HW, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[buf]);
        const bool valid = lt * TILE + row < p.N;
        if (t == seg_first) {
          // a lane's first key of the segment sets its references (invalid lanes only occur in
          // a sequence's partial last tile, which is then the segment's only tile)
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            r[h] = valid ? v[h] * c : -INFINITY;
            l[h] = valid ? 1.f : 0.f;
          }
          continue;
        }
        float dmax = -INFINITY;
#pragma unroll
        for (int h = 0; h < HW; ++h) {
          v[h] = valid ? fmaf(v[h], c, -r[h]) : -INFINITY;  // exponent relative to the reference
          dmax = fmaxf(dmax, v[h]);
        }
        if (__any_sync(0xffffffffu, dmax > REF_SLACK)) {
          // rare: move the reference of the heads that outgrew it (always on a lane's first key)
#pragma unroll
          for (int h = 0; h < HW; ++h) {
            const float d = v[h];
            if (d > REF_SLACK) {
              l[h] = l[h] * fast_exp2(-d) + 1.f;
              r[h] = r[h] + d;
            } else {
              l[h] += fast_exp2(d);
            }
          }
        } else {
#pragma unroll
          for (int h = 0; h < HW; ++h) l[h] += fast_exp2(v[h]);
        }
      }
      // merge the 128 lanes: warp shuffle, then the 4 warps through shared memory
#pragma unroll
      for (int h = 0; h < HW; ++h) {
        float mm = r[h], ll = l[h];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const float m2 = __shfl_xor_sync(0xffffffffu, mm, off);
          const float l2 = __shfl_xor_sync(0xffffffffu, ll, off);
          const float mx = fmaxf(mm, m2);
          const float a1 = mm == -INFINITY ? 0.f : fast_exp2(mm - mx);
          const float a2 = m2 == -INFINITY ? 0.f : fast_exp2(m2 - mx);
          ll = ll * a1 + l2 * a2;
          mm = mx;
        }
        if (lane == 0) { red[wg][wq][h][0] = mm; red[wg][wq][h][1] = ll; }
      }
      named_bar(1 + wg, 128);
      if (wg_tid < HW) {
        float mm = red[wg][0][wg_tid][0], ll = red[wg][0][wg_tid][1];
        for (int w = 1; w < 4; ++w) {
          const float m2 = red[wg][w][wg_tid][0], l2 = red[wg][w][wg_tid][1];
          const float mx = fmaxf(mm, m2);
          const float a1 = mm == -INFINITY ? 0.f : fast_exp2(mm - mx);
          const float a2 = m2 == -INFINITY ? 0.f : fast_exp2(m2 - mx);
          ll = ll * a1 + l2 * a2;
          mm = mx;
        }
        p.ml[(size_t)slot * 2 * H + wg * HW + wg_tid] = mm;
        p.ml[(size_t)slot * 2 * H + H + wg * HW + wg_tid] = ll;
      }
      named_bar(1 + wg, 128);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 128); }
}

// ------------------------------------------------------------------------------------------
// pass 2: exact probabilities, output partials, head-summed scores, histogram
// ------------------------------------------------------------------------------------------
template <int H, int D>
__global__ void __launch_bounds__(NTHREADS, 1)
    dec_pass2_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, DecParams p) {
  static_assert(H == 64 && D == 128, "decode pass 2 is instantiated for 64 heads x 128");
  constexpr int KST = 2, VST = 3;
  constexpr int KT_BYTES = TILE * D * 2;
  constexpr int Q_BYTES = H * D * 2;
  constexpr int P_BYTES = TILE * H * 2;
  constexpr int NKB = D / 64;
  constexpr int NBINS = 2048;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;                           // 1 x Q
  uint8_t* sK = sQ + Q_BYTES;                   // KST x K tile
  uint8_t* sV = sK + KST * KT_BYTES;            // VST x V tile
  uint8_t* sP = sV + VST * KT_BYTES;            // 2 x P^T
  uint32_t* shist = (uint32_t*)(sP + 2 * P_BYTES);
  __shared__ __align__(8) uint64_t k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], s_empty[2],
      p_full[2], p_empty[2], q_full, q_empty, o_full, o_empty;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ __align__(16) float slse[H];
  __shared__ int s_last;
  __shared__ unsigned s_wtot[8];

  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  long long t0, t1;
  tile_range(p, cta, t0, t1);
  const long long limit = p.wait_ns;
  const uint32_t tS = 0, tO = 2 * H;  // TMEM column offsets

  for (int i = threadIdx.x; i < NBINS; i += NTHREADS) shist[i] = 0;
  if (threadIdx.x == 0) {
    for (int i = 0; i < KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < VST; ++i) { mbar_init(&v_full[i], 1); mbar_init(&v_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4); mbar_init(&p_empty[i], 1);
    }
    mbar_init(&q_full, 1); mbar_init(&q_empty, 1);
    mbar_init(&o_full, 1); mbar_init(&o_empty, 4);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, 256); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  griddep_launch_dependents();
  // Launched early (programmatic dependent launch): the producers and the tensor core only read
  // K, V and Q, so they start at once; the softmax warps wait for pass 1 to complete before they
  // read its partials or touch the histogram / counters it cleared.

  // segments are walked from the end of the range backwards, tiles likewise
  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmQ);
      const uint64_t pol = policy_evict_first();
      uint32_t j = 0;
      int seg = 0;
      bool ok = true;
      for (long long t = t1 - 1; t >= t0 && ok; ++seg) {
        const int b = (int)(t / p.tps);
        const long long seg_lo = t0 > (long long)b * p.tps ? t0 : (long long)b * p.tps;
        if (!wait_bar(&q_empty, (seg & 1) ^ 1, limit, &abort_flag, p.st, 201)) { ok = false; break; }
        mbar_expect_tx(&q_full, Q_BYTES);
        for (int kb = 0; kb < NKB; ++kb) tma_load_3d(sQ + kb * (H * 128), &tmQ, &q_full, kb * 64, 0, b);
        for (; t >= seg_lo; --t, ++j) {
          const int lt = (int)(t - (long long)b * p.tps);
          const int s = j % KST;
          if (!wait_bar(&k_empty[s], ((j / KST) & 1) ^ 1, limit, &abort_flag, p.st, 202)) { ok = false; break; }
          mbar_expect_tx(&k_full[s], KT_BYTES);
          for (int kb = 0; kb < NKB; ++kb)
            tma_load_3d_hint(sK + s * KT_BYTES + kb * (TILE * 128), &tmK, &k_full[s], kb * 64, lt * TILE, b, pol);
        }
      }
      if (!ok)
        for (uint32_t jj = (j > KST ? j - KST : 0); jj < j; ++jj) mbar_wait(&k_full[jj % KST], (jj / KST) & 1, limit);
    }
  } else if (warp == 2) {
    if (lane == 0) {
      tma_prefetch_desc(&tmV);
      const uint64_t pol = policy_evict_first();
      uint32_t j = 0;
      bool ok = true;
      for (long long t = t1 - 1; t >= t0 && ok; --t, ++j) {
        const int b = (int)(t / p.tps);
        const int lt = (int)(t - (long long)b * p.tps);
        const int s = j % VST;
        if (!wait_bar(&v_empty[s], ((j / VST) & 1) ^ 1, limit, &abort_flag, p.st, 203)) { ok = false; break; }
        mbar_expect_tx(&v_full[s], KT_BYTES);
        for (int kb = 0; kb < NKB; ++kb)
          tma_load_3d_hint(sV + s * KT_BYTES + kb * (TILE * 128), &tmV, &v_full[s], kb * 64, lt * TILE, b, pol);
      }
      if (!ok)
        for (uint32_t jj = (j > VST ? j - VST : 0); jj < j; ++jj) mbar_wait(&v_full[jj % VST], (jj / VST) & 1, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, H, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16(D, H, 1, 1);
      uint32_t j = 0;
      int seg = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t jj, bool first, int segi) -> bool {
        const int buf = jj & 1, s = jj % VST;
        if (!wait_bar(&p_full[buf], (jj >> 1) & 1, limit, &abort_flag, p.st, 214)) return false;
        if (!wait_bar(&v_full[s], (jj / VST) & 1, limit, &abort_flag, p.st, 215)) return false;
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
        if (!wait_bar(&q_full, seg & 1, limit, &abort_flag, p.st, 211)) { ok = false; break; }
        const uint32_t qaddr = smem_u32(sQ);
        int n_in_seg = 0;
        for (; t >= seg_lo; --t, ++j, ++n_in_seg) {
          const int s = j % KST, buf = j & 1;
          if (!wait_bar(&k_full[s], (j / KST) & 1, limit, &abort_flag, p.st, 212)) { ok = false; break; }
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
        umma_commit(&q_empty);
        if (!issue_pv(j - 1, n_in_seg == 1, seg)) { ok = false; break; }
        umma_commit(&o_full);
      }
    }
  } else if (warp >= SM_WG0) {
    const int wg = (warp - SM_WG0) / 4;    // takes tiles with (j & 1) == wg
    const int wq = (warp - SM_WG0) % 4;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;   // key within the tile == TMEM lane == P^T row
    const int wg_tid = wq * 32 + lane;
    const int all_tid = wg * 128 + wg_tid;  // 0..255 over both warpgroups
    const float c = p.c;
    const int ncand = p.N - p.W > 0 ? p.N - p.W : 0;
    griddep_wait();
    uint32_t j = 0;
    int seg = 0;
    bool ok = true;
    // after a failed wait every later wait returns at once: the loop and named-barrier
    // structure stays identical across all 8 warps, only the work is skipped
    for (long long t = t1 - 1; t >= t0; ++seg) {
      const int b = (int)(t / p.tps);
      const long long seg_lo = t0 > (long long)b * p.tps ? t0 : (long long)b * p.tps;
      const int slot = cta * p.segmax + (b - (int)(t0 / p.tps));
      // the sequence's lse from every pass-1 partial record of it
      if (all_tid < H) {
        const int h = all_tid;
        const int c_lo = cta_of_tile(p, (long long)b * p.tps), c_hi = cta_of_tile(p, (long long)(b + 1) * p.tps - 1);
        float M = -INFINITY, L = 0.f;
        for (int cc = c_lo; cc <= c_hi; ++cc) {
          const long long ct0 = p.total_tiles * cc / p.G;
          const int sl = cc * p.segmax + (b - (int)(ct0 / p.tps));
          const float m = p.ml[(size_t)sl * 2 * H + h], l = p.ml[(size_t)sl * 2 * H + H + h];
          if (!(l > 0.f)) continue;
          const float mx = fmaxf(M, m);
          L = L * (M == -INFINITY ? 0.f : exp2f(M - mx)) + l * exp2f(m - mx);
          M = mx;
        }
        const float lse2 = M + log2f(L);
        slse[h] = lse2;
        if (cta == c_lo) p.lse_out[b * H + h] = lse2 * 0.69314718055994531f;
      }
      named_bar(3, 256);
      const long long n_seg = t - seg_lo + 1;
      for (long long x = 0; x < n_seg; ++x, --t, ++j) {
        if ((int)(j & 1) != wg || !ok) continue;  // the other warpgroup's tile, or unwinding
        const int lt = (int)(t - (long long)b * p.tps);
        const int buf = j & 1;
        if (!warp_wait_bar(&s_full[buf], (j >> 1) & 1, limit, &abort_flag, p.st, 221)) { ok = false; continue; }
        tc_fence_after();
        float v[H];
#pragma unroll
        for (int cc = 0; cc < H / 32; ++cc) {
          float tmp[32];
          tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + tS + buf * H + cc * 32, tmp);
#pragma unroll
          for (int x2 = 0; x2 < 32; ++x2) v[cc * 32 + x2] = tmp[x2];
        }
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[buf]);
        const int key = lt * TILE + row;
        const bool valid = key < p.N;
        float score0 = 0.f, score1 = 0.f;
        uint32_t pk[H / 2];
#pragma unroll
        for (int h = 0; h < H; h += 4) {
          const float4 ls = *reinterpret_cast<const float4*>(&slse[h]);
          const float p0 = valid ? fast_exp2(fmaf(v[h], c, -ls.x)) : 0.f;
          const float p1 = valid ? fast_exp2(fmaf(v[h + 1], c, -ls.y)) : 0.f;
          const float p2 = valid ? fast_exp2(fmaf(v[h + 2], c, -ls.z)) : 0.f;
          const float p3 = valid ? fast_exp2(fmaf(v[h + 3], c, -ls.w)) : 0.f;
          score0 += p0 + p1;
          score1 += p2 + p3;
          pk[h / 2] = pack_bf16x2(p0, p1);
          pk[h / 2 + 1] = pack_bf16x2(p2, p3);
        }
        const float score = score0 + score1;
        if (!warp_wait_bar(&p_empty[buf], ((j >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 222)) { ok = false; continue; }
        const uint32_t prow = smem_u32(sP + buf * P_BYTES);
#pragma unroll
        for (int ch = 0; ch < H / 8; ++ch)
          st_shared_v4(prow + sw128_off(row, ch), pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[buf]);
        const bool is_cand = valid && key < ncand;
        if (is_cand) p.sc[(size_t)b * ncand + key] = score;
        const unsigned bin = (__float_as_uint(score) >> 20) & (NBINS - 1);
        const unsigned act = __ballot_sync(0xffffffffu, is_cand);
        if (is_cand) {
          const unsigned peers = __match_any_sync(act, bin);
          if ((int)(__ffs(peers) - 1) == lane) atomicAdd(&shist[bin], (unsigned)__popc(peers));
        }
      }
      // segment done: warpgroup 0 fetches O^T (lane = output column d, one TMEM column per head)
      if (wg == 0 && ok) {
        if (!warp_wait_bar(&o_full, seg & 1, limit, &abort_flag, p.st, 223)) { ok = false; }
        if (ok) {
          tc_fence_after();
          float* dst = p.opart + (size_t)slot * H * D;
#pragma unroll
          for (int cc = 0; cc < H / 32; ++cc) {
            float o[32];
            tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + tO + cc * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int x2 = 0; x2 < 32; ++x2) dst[(cc * 32 + x2) * D + row] = o[x2];
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&o_empty);
        }
      }
      // flush this sequence's histogram (both warpgroups are done with the segment)
      named_bar(3, 256);
      for (int i = all_tid; i < NBINS; i += 256) {
        const uint32_t cnt = shist[i];
        if (cnt) { atomicAdd(&p.hist[(size_t)b * NBINS + i], cnt); shist[i] = 0; }
      }
      __threadfence();
      named_bar(3, 256);
      // the last CTA to finish this sequence finds the bin of its k-th largest score
      if (all_tid == 0) {
        const int c_lo = cta_of_tile(p, (long long)b * p.tps), c_hi = cta_of_tile(p, (long long)(b + 1) * p.tps - 1);
        s_last = atomicAdd(&p.seq_done[b], 1) == c_hi - c_lo;
      }
      named_bar(3, 256);
      if (s_last) {
        __threadfence();
        int* meta = p.meta + b * 8;
        const int K = p.K_sel;
        if (ncand <= K || K == 0) {
          if (all_tid == 0) {
            meta[0] = K == 0 ? NBINS : -1;  // -1: every older token; NBINS: none
            meta[1] = K == 0 ? 0 : ncand;
            meta[2] = 0; meta[3] = 0; meta[4] = 0;
          }
        } else {
          // thread i owns bins hi..hi-7 (descending); block-inclusive scan of their counts
          const int hi = NBINS - 1 - 8 * all_tid;
          unsigned cnt8[8], local = 0;
#pragma unroll
          for (int x = 0; x < 8; ++x) { cnt8[x] = __ldcg(&p.hist[(size_t)b * NBINS + hi - x]); local += cnt8[x]; }
          unsigned incl = local;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned nb = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nb;
          }
          const int wv = all_tid >> 5;
          if (lane == 31) s_wtot[wv] = incl;
          named_bar(3, 256);
          unsigned add = 0;
          for (int x = 0; x < wv; ++x) add += s_wtot[x];
          incl += add;
          const unsigned excl = incl - local;
          if (excl < (unsigned)K && incl >= (unsigned)K) {
            unsigned run = excl;
            for (int x = 0; x < 8; ++x) {
              if (run + cnt8[x] >= (unsigned)K) {
                meta[0] = hi - x; meta[1] = (int)run; meta[2] = (int)(K - run); meta[3] = 0; meta[4] = 0;
                break;
              }
              run += cnt8[x];
            }
          }
        }
      }
      named_bar(3, 256);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 256); }
}

// ------------------------------------------------------------------------------------------
// host launcher
// ------------------------------------------------------------------------------------------
size_t pass1_smem_bytes(int H, int D) { return 1024 + 2 * (size_t)H * D * 2 + 5 * (size_t)TILE * D * 2; }
size_t pass2_smem_bytes(int H, int D) {
  return 1024 + (size_t)H * D * 2 + 5 * (size_t)TILE * D * 2 + 2 * (size_t)TILE * H * 2 + 2048 * 4;
}

cudaError_t launch_decode_attn(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                               const DecParams& p, cudaStream_t stream) {
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
  cudaError_t e;
  {
    LaunchScope ls("dec_pass2", stream);
    e = launch_k(dec_pass2_kernel<H, D>, dim3(p.G), dim3(NTHREADS), pass2_smem_bytes(H, D), stream, true, tmK, tmV,
                 tmQ, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace dec
}  // namespace hs2
