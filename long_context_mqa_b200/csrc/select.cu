// Exact top-k over a per-sequence score vector (decode path), ties to the lower index.
//
//  0. (same kernel as 1) the decode output: per sequence, the sum of the per-segment output
//                 partials of the CTAs whose tile ranges cover it, rounded to bf16.
//  1. threshold : from the 2048-bin histogram of score bits 30..20 (filled by decode pass 2),
//                 find the bin beta that holds the k-th largest score; `above` = number of
//                 scores in higher bins, `need` = k - above.
//  2. collect   : every score in a bin above beta is selected outright; scores in bin beta
//                 become 64-bit keys (score bits << 32 | ~index) -- unique, and larger key ==
//                 higher score, then lower index.
//  3. final     : MSB-first 8-bit radix select of the `need` largest boundary keys, then the
//                 forced window is appended and the <= 2048 indices are sorted ascending.
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace sel {

constexpr int NT = 1024;

// inclusive block scan (sum) of one value per thread, NT threads
__device__ __forceinline__ unsigned block_incl_scan(unsigned v, unsigned* warp_tot) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_tot[w] = v;
  __syncthreads();
  if (w == 0) {
    unsigned t = warp_tot[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned n = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += n;
    }
    warp_tot[lane] = t;
  }
  __syncthreads();
  if (w > 0) v += warp_tot[w - 1];
  __syncthreads();
  return v;
}

__global__ void __launch_bounds__(NT) sel_threshold_kernel(SelParams p) {
  const int b = blockIdx.x, tid = threadIdx.x;
  __shared__ unsigned h[NBINS];
  __shared__ unsigned wt[32];
  int* meta = p.meta + b * META;
  {
    // decode output: CTAs c_lo..c_hi cover this sequence's tiles (contiguous split of the
    // flattened tile space); slot = c * segmax + (b - first sequence of c)
    const long long x_lo = (long long)b * p.tps, x_hi = (long long)(b + 1) * p.tps - 1;
    const int c_lo = (int)(((x_lo + 1) * p.G - 1) / p.total_tiles);
    const int c_hi = (int)(((x_hi + 1) * p.G - 1) / p.total_tiles);
    for (int e = tid; e < p.H * p.D; e += NT) {
      float acc = 0.f;
      for (int c = c_lo; c <= c_hi; ++c) {
        const long long ct0 = p.total_tiles * c / p.G;
        const int slot = c * p.segmax + (b - (int)(ct0 / p.tps));
        acc += p.opart[(size_t)slot * p.H * p.D + e];
      }
      p.out[(size_t)b * p.H * p.D + e] = __float2bfloat16_rn(acc);
    }
  }
  if (tid == 0) { meta[3] = 0; meta[4] = 0; }
  if (p.K == 0) {  // nothing is chosen by score
    if (tid == 0) { meta[0] = NBINS; meta[1] = 0; meta[2] = 0; }
    return;
  }
  if (p.ncand <= p.K) {  // every older token is selected
    if (tid == 0) { meta[0] = -1; meta[1] = p.ncand; meta[2] = 0; }
    return;
  }
  for (int i = tid; i < NBINS; i += NT) h[i] = p.hist[(size_t)b * NBINS + i];
  __syncthreads();
  const int hi = NBINS - 1 - 2 * tid;  // this thread's bins: hi, hi - 1 (descending order)
  const unsigned local = h[hi] + h[hi - 1];
  const unsigned incl = block_incl_scan(local, wt);
  const unsigned excl = incl - local;
  const unsigned K = (unsigned)p.K;
  if (excl < K && incl >= K) {
    if (excl + h[hi] >= K) { meta[0] = hi; meta[1] = (int)excl; meta[2] = (int)(K - excl); }
    else { meta[0] = hi - 1; meta[1] = (int)(excl + h[hi]); meta[2] = (int)(K - excl - h[hi]); }
  }
}

__global__ void __launch_bounds__(NT) sel_collect_kernel(SelParams p) {
  const int b = blockIdx.y;
  int* meta = p.meta + b * META;
  const int beta = meta[0];
  const int lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const float* sc = p.sc + (size_t)b * p.ncand;
  const int stride = gridDim.x * NT;
  const int n_round = (p.ncand + 31) & ~31;
  for (int j = blockIdx.x * NT + threadIdx.x; j < n_round; j += stride) {
    int bin = -2;
    uint32_t bits = 0;
    if (j < p.ncand) {
      bits = __float_as_uint(sc[j]);
      bin = (int)((bits >> 20) & (NBINS - 1));
    }
    const bool up = bin > beta;
    const bool eq = bin == beta;
    const unsigned mu = __ballot_sync(0xffffffffu, up);
    const unsigned me = __ballot_sync(0xffffffffu, eq);
    if (mu) {
      int base = 0;
      const int leader = __ffs(mu) - 1;
      if (lane == leader) base = atomicAdd(&meta[3], __popc(mu));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (up) {
        const int pos = base + __popc(mu & lt_mask);
        if (pos < p.K) p.above[(size_t)b * p.K + pos] = j;
        else report_status(p.st, kStatusBounds, 301);
      }
    }
    if (me) {
      int base = 0;
      const int leader = __ffs(me) - 1;
      if (lane == leader) base = atomicAdd(&meta[4], __popc(me));
      base = __shfl_sync(0xffffffffu, base, leader);
      if (eq) {
        const int pos = base + __popc(me & lt_mask);
        p.bnd[(size_t)b * p.ncand + pos] = ((unsigned long long)bits << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)j);
      }
    }
  }
}

__global__ void __launch_bounds__(NT) sel_final_kernel(SelParams p) {
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  __shared__ int list[2048];
  __shared__ unsigned dh[256];
  __shared__ unsigned long long s_prefix, s_mask;
  __shared__ int s_need, s_cnt;
  const int* meta = p.meta + b * META;
  const int n_above = meta[1];
  const int need = meta[2];
  const int n_bnd = meta[4];
  const unsigned long long* bnd = p.bnd + (size_t)b * p.ncand;
  for (int i = tid; i < 2048; i += NT) list[i] = 0x7FFFFFFF;
  __syncthreads();
  for (int i = tid; i < n_above && i < p.K; i += NT) list[i] = p.above[(size_t)b * p.K + i];
  if (tid == 0) { s_prefix = 0; s_mask = 0; s_need = need; s_cnt = 0; }
  __syncthreads();
  if (need > 0) {
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += NT) dh[i] = 0;
      __syncthreads();
      const unsigned long long prefix = s_prefix, mask = s_mask;
      for (int i = tid; i < n_bnd; i += NT) {
        const unsigned long long key = bnd[i];
        if ((key & mask) == prefix) atomicAdd(&dh[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (w == 0) {
        // lane l owns digits 255-8l .. 248-8l (descending)
        unsigned cnt[8], tot = 0;
#pragma unroll
        for (int x = 0; x < 8; ++x) { cnt[x] = dh[255 - 8 * lane - x]; tot += cnt[x]; }
        unsigned incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        const unsigned excl = incl - tot;
        const unsigned k = (unsigned)s_need;
        if (excl < k && incl >= k) {
          unsigned run = excl;
          for (int x = 0; x < 8; ++x) {
            if (run + cnt[x] >= k) {
              const unsigned digit = 255u - 8u * lane - x;
              s_need = (int)(k - run);
              s_prefix = prefix | ((unsigned long long)digit << shift);
              s_mask = mask | (255ull << shift);
              break;
            }
            run += cnt[x];
          }
        }
      }
      __syncthreads();
    }
    // s_prefix is now the exact key of the need-th largest boundary entry
    const unsigned long long thr = s_prefix;
    for (int i = tid; i < n_bnd; i += NT) {
      const unsigned long long key = bnd[i];
      if (key >= thr) {
        const int pos = atomicAdd(&s_cnt, 1);
        if (n_above + pos < 2048) list[n_above + pos] = (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
      }
    }
    __syncthreads();
  }
  const int n_top = n_above + (need > 0 ? s_cnt : 0);
  const int wlen = p.N < p.W ? p.N : p.W;
  for (int i = tid; i < wlen; i += NT)
    if (n_top + i < 2048) list[n_top + i] = p.N - wlen + i;
  const int total = n_top + wlen;
  const int expect = p.N < p.S ? p.N : p.S;
  if (tid == 0 && total != expect) report_status(p.st, kStatusBounds, 302);
  __syncthreads();
  // bitonic sort, ascending, 2048 slots
  for (int k = 2; k <= 2048; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      const int i = 2 * tid - (tid & (j - 1));
      const int l = i + j;
      const int a = list[i], c = list[l];
      const bool asc = (i & k) == 0;
      if ((a > c) == asc) { list[i] = c; list[l] = a; }
      __syncthreads();
    }
  }
  for (int i = tid; i < p.S; i += NT) p.idx[(size_t)b * p.S + i] = (i < total && i < 2048) ? list[i] : -1;
}

cudaError_t launch_select(const SelParams& p, cudaStream_t stream) {
  {
    LaunchScope ls("sel_threshold", stream);
    sel_threshold_kernel<<<p.B, NT, 0, stream>>>(p);
  }
  if (p.ncand > 0) {
    int blocks = (p.ncand + NT - 1) / NT;
    if (blocks > 64) blocks = 64;
    LaunchScope ls("sel_collect", stream);
    sel_collect_kernel<<<dim3(blocks, p.B), NT, 0, stream>>>(p);
  }
  {
    LaunchScope ls("sel_final", stream);
    sel_final_kernel<<<p.B, NT, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace sel
}  // namespace hs2
