// HySparse (v1) block-level selection of the decode path: for the one query of each sequence
// (position t), the n_blocks blocks of `block` consecutive tokens with the largest block score,
// ties to the lower block, plus the `window` most recent tokens as a separate branch
// (arex-research.com article "小米 MiMo 负责人罗福利公开 MiMo-V3 核心架构 HySparse2", section
// "外层 KV Bridging，内层 KV Reuse": HySparse picks its 1,024 global tokens in 64-token blocks and
// keeps a gated 128-token sliding-window branch beside them). The block score is the sum of the
// token scores score(t, j) = sum_h p_h(t, j) of the block's tokens at or before t; every block
// starting at or before t competes (the window branch is separate, so recent blocks compete too).
//
// It runs after the fused decode kernel (decode.cu), which, given a buffer for them, stores for
// every group of 32 consecutive keys the per-head sums P'_gh = sum over the group of p'_jh
// (p' = exp2(s c - lse2') against its sampled reference) and, per head, the exact totals
// L'_h = sum_j p'_jh. The exact probability of key j under head h is p'_jh / L'_h, so block J
// (groups 2J and 2J + 1) scores exactly
//   score_J = sum_h (P'_{2J,h} + P'_{2J+1,h}) / L'_h,
// with no second pass over K.
//  1. score (a warp per block, many CTAs): score_J for every block of every sequence, the two
//     groups and the heads summed in a fixed order. Extra CTAs of the same launch write the decode
//     output (sum of the decode kernel's records / L'), and one thread re-arms the decode kernel's
//     grid barrier.
//  2. final (one CTA per sequence): the n_blocks largest blocks by the unique 64-bit keys
//     (score bits << 32 | ~block: larger key == higher score, then lower block), an MSB-first
//     8-bit radix select; their tokens <= t ascending into the first n_blocks * block slots of the
//     row (-1 after), the window t - window + 1 .. t into the last `window` slots.
#include "combine.cuh"
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace blk {

constexpr int NT = 1024;
constexpr int WARPS = NT / 32;

__global__ void __launch_bounds__(NT) blk_score_kernel(BlkParams p, int score_ctas_per_seq) {
  griddep_wait();
  griddep_launch_dependents();
  // both decode launches are complete: re-arm their grid barrier for the next step
  if (blockIdx.x == 0 && threadIdx.x == 0) *(volatile unsigned*)p.gbar = 0u;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int n_score = p.B * score_ctas_per_seq;
  if ((int)blockIdx.x >= n_score) {
    // the decode output (independent of the selection), a warp per head: WARPS heads per CTA
    const int oc = blockIdx.x - n_score, per_seq = (p.H + WARPS - 1) / WARPS;
    const int h = (oc % per_seq) * WARPS + w;
    if (h < p.H)
      combine_decode_output(p.opart, p.lsum, p.oscale, p.out, p.H, p.D, p.sch, p.st, oc / per_seq, h, lane);
    return;
  }
  const int b = blockIdx.x / score_ctas_per_seq;
  const int J = (blockIdx.x % score_ctas_per_seq) * WARPS + w;
  const int t = p.sch.seq_len[b] - 1;
  const int nb = t / p.BLK + 1;  // blocks meeting 0..t
  if (J >= nb || p.H != 64) return;
  // lane l: heads 2l and 2l + 1 of both groups of the block (a group past t holds p' = 0 for
  // every key after t, and the second group of the last block may not exist at all)
  const float2 L = reinterpret_cast<const float2*>(p.lsum + (size_t)b * p.H)[lane];
  const float* g0 = p.blk_part + ((size_t)b * p.blk_groups + 2 * (size_t)J) * p.H;
  const float2 a = __ldcg(reinterpret_cast<const float2*>(g0) + lane);
  float2 c = make_float2(0.f, 0.f);
  if (2 * J + 1 <= t / 32) c = __ldcg(reinterpret_cast<const float2*>(g0 + p.H) + lane);
  float s = (a.x + c.x) / L.x + (a.y + c.y) / L.y;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) p.bsc[(size_t)b * p.max_blocks + J] = s;
}

__global__ void __launch_bounds__(NT) blk_final_kernel(BlkParams p) {
  griddep_wait();
  griddep_launch_dependents();
  __shared__ unsigned hist[256];
  __shared__ unsigned long long s_prefix, s_mask;
  __shared__ int s_need, s_exact, s_n;
  __shared__ int s_sel[32];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int t = p.sch.seq_len[b] - 1;
  const int nb = t / p.BLK + 1;
  const float* bsc = p.bsc + (size_t)b * p.max_blocks;
  auto key_of = [&](int J) {  // larger key == higher score, then lower block
    return ((unsigned long long)__float_as_uint(bsc[J]) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)J);
  };
  if (tid == 0) { s_prefix = 0ull; s_mask = 0ull; s_need = p.NB; s_exact = 0; s_n = 0; }
  __syncthreads();
  unsigned long long thr = 0ull, fmask = 0ull;  // every block is chosen when at most NB exist
  if (nb > p.NB) {
    // MSB-first 8-bit radix select of the NB largest keys (scores are >= 0, so a score's bits
    // order as its value); stops as soon as a digit's bucket holds exactly the remaining need
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += NT) hist[i] = 0u;
      __syncthreads();
      const unsigned long long prefix = s_prefix, mask = s_mask;
      for (int J = tid; J < nb; J += NT) {
        const unsigned long long k = key_of(J);
        if ((k & mask) == prefix) atomicAdd(&hist[(k >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (w == 0) {
        // lane l owns digits 255 - 8l .. 248 - 8l (descending)
        unsigned cnt[8], tot = 0;
#pragma unroll
        for (int x = 0; x < 8; ++x) { cnt[x] = hist[255 - 8 * lane - x]; tot += cnt[x]; }
        unsigned incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const unsigned excl = incl - tot, k = (unsigned)s_need;
        if (excl < k && incl >= k) {
          unsigned run = excl;
          for (int x = 0; x < 8; ++x) {
            if (run + cnt[x] >= k) {
              s_need = (int)(k - run);
              s_prefix = prefix | ((unsigned long long)(255u - 8u * lane - x) << shift);
              s_mask = mask | (255ull << shift);
              s_exact = run + cnt[x] == k;  // the whole bucket is taken: no further digit needed
              break;
            }
            run += cnt[x];
          }
        }
      }
      __syncthreads();
      if (s_exact) break;
    }
    thr = s_prefix;
    fmask = s_mask;
  }
  // the chosen blocks: keys whose masked prefix is >= the threshold (exactly NB of them, or all)
  for (int J = tid; J < nb; J += NT) {
    if ((key_of(J) & fmask) >= thr) {
      const int at = atomicAdd(&s_n, 1);
      if (at < 32) s_sel[at] = J;
    }
  }
  __syncthreads();
  const int n_sel = s_n < 32 ? s_n : 32;
  if (tid == 0) {
    if (s_n != (nb <= p.NB ? nb : p.NB)) report_status(p.st, kStatusBounds, 521);
    for (int i = 1; i < n_sel; ++i) {  // ascending block order (at most n_blocks entries)
      const int x = s_sel[i];
      int k = i - 1;
      while (k >= 0 && s_sel[k] > x) { s_sel[k + 1] = s_sel[k]; --k; }
      s_sel[k + 1] = x;
    }
  }
  __syncthreads();
  int32_t* out = p.idx + (size_t)b * p.S;
  const int nblk_slots = p.NB * p.BLK;
  for (int s = tid; s < p.S; s += NT) {
    int tok = -1;
    if (s < nblk_slots) {
      const int k = s / p.BLK;
      if (k < n_sel) {
        const int j = s_sel[k] * p.BLK + s % p.BLK;
        tok = j <= t ? j : -1;
      }
    } else {
      const int lo = t - p.W + 1 > 0 ? t - p.W + 1 : 0;
      const int j = lo + (s - nblk_slots);
      tok = j <= t ? j : -1;
    }
    out[s] = tok;
  }
}

cudaError_t launch_block_select(const BlkParams& p, cudaStream_t stream) {
  cudaError_t e;
  {
    LaunchScope ls("blk_score", stream);
    const int score_ctas = (p.max_blocks + WARPS - 1) / WARPS;
    const int per_seq = (p.H + WARPS - 1) / WARPS;
    e = launch_k(blk_score_kernel, dim3(p.B * score_ctas + p.B * per_seq), dim3(NT), 0, stream, true, p, score_ctas);
  }
  if (e != cudaSuccess) return e;
  {
    LaunchScope ls("blk_final", stream);
    e = launch_k(blk_final_kernel, dim3(p.B), dim3(NT), 0, stream, true, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace blk
}  // namespace hs2
