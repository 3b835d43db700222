// Exact top-k over a per-sequence score vector (decode path), ties to the lower index.
//
//  1. threshold : (done by decode pass 2) from the 2048-bin histogram of score bits 30..20,
//                 the bin beta that holds the k-th largest score; `above` = number of scores in
//                 higher bins, `need` = k - above.
//  2. collect   : every score in a bin above beta is selected outright; scores in bin beta
//                 become 64-bit keys (score bits << 32 | ~index) -- unique, and larger key ==
//                 higher score, then lower index. Extra CTAs of the same launch produce the
//                 decode output: per (sequence, head), the sum of the per-segment output partials
//                 of the CTAs whose tile ranges cover the sequence, rounded to bf16.
//  3. final     : MSB-first 8-bit radix select of the `need` largest boundary keys, then the
//                 forced window is appended and the <= 2048 indices are sorted ascending.
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace sel {

constexpr int NT = 1024;

__device__ __forceinline__ void collect_one(const SelParams& p, int b, int* meta, int beta, int j, float score,
                                            bool in_range, unsigned lane, unsigned lt_mask) {
  int bin = -2;
  uint32_t bits = 0;
  if (in_range) {
    bits = __float_as_uint(score);
    bin = (int)((bits >> 20) & (NBINS - 1));
  }
  const bool up = bin > beta;
  const bool eq = bin == beta;
  const unsigned mu = __ballot_sync(0xffffffffu, up);
  const unsigned me = __ballot_sync(0xffffffffu, eq);
  if (mu) {
    int base = 0;
    const int leader = __ffs(mu) - 1;
    if ((int)lane == leader) base = atomicAdd(&meta[3], __popc(mu));
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
    if ((int)lane == leader) base = atomicAdd(&meta[4], __popc(me));
    base = __shfl_sync(0xffffffffu, base, leader);
    if (eq) {
      const int pos = base + __popc(me & lt_mask);
      p.bnd[(size_t)b * p.ncand + pos] = ((unsigned long long)bits << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)j);
    }
  }
}

// blockIdx.x < n_collect: every score of every older token -- above the boundary bin ->
// selected; in it -> 64-bit key. blockIdx.x >= n_collect: output of head (blockIdx.x - n_collect).
__global__ void __launch_bounds__(256) sel_collect_kernel(SelParams p, int n_collect) {
  griddep_wait();
  griddep_launch_dependents();
  const int b = blockIdx.y;
  if ((int)blockIdx.x >= n_collect) {
    // CTAs c_lo..c_hi cover sequence b's tiles (contiguous split of the flattened tile space);
    // slot = c * segmax + (b - first sequence of c)
    __shared__ int slot_off[256];  // one entry per covering CTA (at most one CTA per SM)
    __shared__ int n_slots;
    const int h = blockIdx.x - n_collect;
    if (threadIdx.x == 0) {
      const long long x_lo = (long long)b * p.tps, x_hi = (long long)(b + 1) * p.tps - 1;
      const int c_lo = (int)(((x_lo + 1) * p.G - 1) / p.total_tiles);
      const int c_hi = (int)(((x_hi + 1) * p.G - 1) / p.total_tiles);
      int n = 0;
      for (int c = c_lo; c <= c_hi && n < 256; ++c, ++n) {
        const long long ct0 = p.total_tiles * c / p.G;
        slot_off[n] = c * p.segmax + (b - (int)(ct0 / p.tps));
      }
      n_slots = c_hi - c_lo + 1;
    }
    __syncthreads();
    if (n_slots > 256) {  // more covering CTAs than SMs on any sm_100 part: not a valid split
      if (threadIdx.x == 0) report_status(p.st, kStatusBounds, 303);
      return;
    }
    for (int d = threadIdx.x; d < p.D; d += blockDim.x) {
      float acc = 0.f;
#pragma unroll 8
      for (int i = 0; i < n_slots; ++i) acc += p.opart[((size_t)slot_off[i] * p.H + h) * p.D + d];
      p.out[((size_t)b * p.H + h) * p.D + d] = __float2bfloat16_rn(acc);
    }
    return;
  }
  int* meta = p.meta + b * META;
  const int beta = meta[0];
  const unsigned lane = threadIdx.x & 31;
  const unsigned lt_mask = (1u << lane) - 1u;
  const float* sc = p.sc + (size_t)b * p.ncand;
  const int stride = n_collect * 256 * 4;
  const int n_round = ((p.ncand + 127) / 128) * 128;
  // four consecutive scores per thread per step (16-byte loads when the row is aligned)
  const bool vec = ((reinterpret_cast<uintptr_t>(sc) & 15u) == 0);
  for (int j0 = (blockIdx.x * 256 + threadIdx.x) * 4; j0 < n_round; j0 += stride) {
    float v[4] = {0.f, 0.f, 0.f, 0.f};
    if (vec && j0 + 3 < p.ncand) {
      const float4 f = *reinterpret_cast<const float4*>(sc + j0);
      v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    } else {
      for (int x = 0; x < 4; ++x)
        if (j0 + x < p.ncand) v[x] = sc[j0 + x];
    }
#pragma unroll
    for (int x = 0; x < 4; ++x) collect_one(p, b, meta, beta, j0 + x, v[x], j0 + x < p.ncand, lane, lt_mask);
  }
}

__global__ void __launch_bounds__(NT) sel_final_kernel(SelParams p) {
  griddep_wait();
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
    // bits on which every boundary key agrees need no pass: start at the highest differing bit
    __shared__ unsigned long long s_and, s_or;
    if (tid == 0) { s_and = ~0ull; s_or = 0ull; }
    __syncthreads();
    unsigned long long a_loc = ~0ull, o_loc = 0ull;
    for (int i = tid; i < n_bnd; i += NT) { const unsigned long long key = bnd[i]; a_loc &= key; o_loc |= key; }
    for (int o = 16; o > 0; o >>= 1) {
      a_loc &= __shfl_xor_sync(0xffffffffu, a_loc, o);
      o_loc |= __shfl_xor_sync(0xffffffffu, o_loc, o);
    }
    if (lane == 0) { atomicAnd(&s_and, a_loc); atomicOr(&s_or, o_loc); }
    __syncthreads();
    const unsigned long long diff = s_and ^ s_or;
    const int top = diff ? 63 - __clzll((long long)diff) : 0;  // highest differing bit
    if (tid == 0) { s_prefix = s_and & ~((top >= 63) ? 0ull : ((2ull << top) - 1ull)); s_mask = (top >= 63) ? 0ull : ~((2ull << top) - 1ull); }
    __syncthreads();
    // 8-bit digit windows [shift, shift + 8) from the top down; the last window is clamped at
    // bit 0 (its bits above the previous window's are already fixed in the prefix)
    for (int sh_raw = top - 7;; sh_raw -= 8) {
      const int shift = sh_raw < 0 ? 0 : sh_raw;
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
      if (shift == 0) break;
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
  cudaError_t e;
  {
    int n_collect = (p.ncand + 1023) / 1024;  // 256 threads x 4 scores
    if (n_collect > 128) n_collect = 128;
    if (n_collect < 1) n_collect = 1;
    LaunchScope ls("sel_collect", stream);
    e = launch_k(sel_collect_kernel, dim3(n_collect + p.H, p.B), dim3(256), 0, stream, true, p, n_collect);
  }
  if (e != cudaSuccess) return e;
  {
    LaunchScope ls("sel_final", stream);
    e = launch_k(sel_final_kernel, dim3(p.B), dim3(NT), 0, stream, true, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sel
}  // namespace hs2
