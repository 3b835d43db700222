// HySparse (v1) block-level selection of the decode path: for the one query of each sequence
// (position t), the n_blocks blocks of `block` consecutive tokens with the largest block score,
// ties to the lower block, plus the `window` most recent tokens as a separate branch
// (arex-research.com article "小米 MiMo 负责人罗福利公开 MiMo-V3 核心架构 HySparse2", section
// "外层 KV Bridging，内层 KV Reuse": HySparse picks its 1,024 global tokens in 64-token blocks and
// keeps a gated 128-token sliding-window branch beside them). The block score is the sum of the
// token scores score(t, j) = sum_h p_h(t, j) of the block's tokens at or before t; every block
// starting at or before t competes (the window branch is separate, so recent blocks compete too).
//
// It runs after the fused decode kernel (decode.cu), which leaves for every older token j < t -
// window + 1 a bounded score score'_j = sum_h p'_jh (p' = exp2(s c - lse2'), the sampled
// reference) and, per head, the exact totals L'_h = sum_j p'_jh. The true score of token j is
// sum_h p'_jh / L'_h, so a block of such tokens has score'-sum S'_J with
//   S'_J / max L' <= score_J <= S'_J / min L'.
//  1. bound   (one CTA per sequence): S'_J of every block wholly among the older tokens, the
//              n_blocks-th largest of them by an 8-bit MSB-first radix select; a block whose upper
//              bound is below the n_blocks-th largest lower bound cannot be chosen. The others,
//              and the (at most three) blocks that reach into the window region, whose tokens
//              have no stored score, are the candidates. Extra CTAs of the same launch write the
//              decode output (sum of the decode kernel's records / L'), and CTA 0 re-arms the
//              decode kernel's grid barrier.
//  2. rescore (persistent): exact scores of the candidates' tokens (their K rows gathered, S^T =
//              K Q^T on tcgen05, sum_h exp2(s c - lse2_h) with the exact lse), summed per block in
//              a fixed order.
//  3. final   (one CTA per sequence): the n_blocks largest candidates by (exact score, then lower
//              block), their tokens <= t ascending into the first n_blocks * block slots of the
//              row (-1 after), the window t - window + 1 .. t into the last `window` slots.
#include "combine.cuh"
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace blk {

constexpr int NT = 1024;
// relative slack of the bounds: covers the rounding of the fp32 sums behind S' and L' and the
// difference between the decode kernel's logits and the re-score's (both fp32 accumulations)
constexpr float kSlack = 1e-4f;

__device__ __forceinline__ float block_sum64(const float* src, bool vec) {
  float s = 0.f;
  if (vec) {
#pragma unroll
    for (int x = 0; x < 16; ++x) {
      const float4 f = __ldcg(reinterpret_cast<const float4*>(src) + x);
      s += f.x; s += f.y; s += f.z; s += f.w;
    }
  } else {
#pragma unroll 8
    for (int x = 0; x < 64; ++x) s += __ldcg(src + x);
  }
  return s;
}

__global__ void __launch_bounds__(NT) blk_bound_kernel(BlkParams p) {
  griddep_wait();
  griddep_launch_dependents();
  // both decode launches are complete: re-arm their grid barrier for the next step
  if (blockIdx.x == 0 && threadIdx.x == 0) *(volatile unsigned*)p.gbar = 0u;
  if ((int)blockIdx.x >= p.B) {
    // the decode output (independent of the selection), a warp per head: NT / 32 heads per CTA
    const int oc = blockIdx.x - p.B, per_seq = (p.H + NT / 32 - 1) / (NT / 32);
    const int h = (oc % per_seq) * (NT / 32) + (int)(threadIdx.x >> 5);
    if (h < p.H)
      combine_decode_output(p.opart, p.lsum, p.oscale, p.out, p.H, p.D, p.sch, p.st, oc / per_seq, h,
                            threadIdx.x & 31);
    return;
  }
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix, s_mask, s_need, s_n;
  __shared__ float s_lmin, s_lmax;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int n_b = p.sch.seq_len[b];
  const int t = n_b - 1;
  const int nb = t / p.BLK + 1;                  // blocks meeting 0..t
  const int nc = n_b - p.W > 0 ? n_b - p.W : 0;  // older tokens (with a stored score')
  const int nfull = p.BLK == 64 ? nc / 64 : 0;   // blocks wholly among them
  int* cand = p.cand + (size_t)b * p.max_blocks;
  float* spb = p.bsc + (size_t)b * p.max_blocks;  // S' of the full blocks (the exact scores later)
  if (nb > p.max_blocks) {
    if (tid == 0) { report_status(p.st, kStatusBounds, 501); p.cnt[b] = 0; }
    return;
  }
  if (nb <= p.NB || nfull < p.NB) {
    // every block is a candidate (at most n_blocks of them, or too few with a stored bound)
    for (int j = tid; j < nb; j += NT) cand[j] = j;
    if (tid == 0) p.cnt[b] = nb;
    return;
  }
  if (w == 0) {
    float mn = INFINITY, mx = 0.f;
    for (int h = lane; h < p.H; h += 32) {
      const float L = p.lsum[b * p.H + h];
      mn = fminf(mn, L);
      mx = fmaxf(mx, L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    }
    if (lane == 0) { s_lmin = mn; s_lmax = mx; s_prefix = 0u; s_mask = 0u; s_need = (unsigned)p.NB; s_n = 0u; }
  }
  const float* sc = p.sc + (size_t)b * p.ncand;
  const bool vec = (reinterpret_cast<uintptr_t>(sc) & 15u) == 0;
  for (int j = tid; j < nfull; j += NT) spb[j] = block_sum64(sc + (size_t)j * 64, vec);
  __syncthreads();
  // the n_blocks-th largest S' (scores are >= 0, so their bit patterns order as the values)
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += NT) hist[i] = 0u;
    __syncthreads();
    const unsigned prefix = s_prefix, mask = s_mask;
    for (int j = tid; j < nfull; j += NT) {
      const unsigned u = __float_as_uint(spb[j]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
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
      const unsigned excl = incl - tot, k = s_need;
      if (excl < k && incl >= k) {
        unsigned run = excl;
        for (int x = 0; x < 8; ++x) {
          if (run + cnt[x] >= k) {
            s_need = k - run;
            s_prefix = prefix | ((255u - 8u * lane - x) << shift);
            s_mask = mask | (255u << shift);
            break;
          }
          run += cnt[x];
        }
      }
    }
    __syncthreads();
  }
  const float kth = __uint_as_float(s_prefix);
  const float rho = s_lmax > 0.f ? s_lmin / s_lmax : 0.f;
  const float tau = kth * rho * ((1.f - kSlack) / (1.f + kSlack));
  // candidates: full blocks with S' >= tau (one list update per warp), then the blocks that
  // reach into the window region
  for (int j0 = 0; j0 < nb; j0 += NT) {
    const int j = j0 + tid;
    const bool take = j < nb && (j >= nfull || spb[j] >= tau);
    const unsigned m = __ballot_sync(0xffffffffu, take);
    unsigned base = 0;
    if (lane == 0 && m) base = atomicAdd(&s_n, (unsigned)__popc(m));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (take) cand[base + __popc(m & ((1u << lane) - 1u))] = j;
  }
  __syncthreads();
  if (tid == 0) p.cnt[b] = (int)s_n;
}

__global__ void __launch_bounds__(128) blk_rescore_kernel(BlkParams p) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int H = 64, D = 128, TILE = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;              // [64 heads][128] K-major SW128 (two 64-column blocks)
  uint8_t* sK = smem + H * D * 2;  // [128 keys][128] K-major SW128
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ __align__(16) float s_nl[H];  // -lse2 of the current sequence
  __shared__ float wsum[4];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) { mbar_init(&mma_bar, 1); fence_mbar_init(); }
  if (warp == 0) { tmem_alloc(&tmem_base, 64); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const float c = p.c;
  int cur_b = -1;
  uint32_t phase = 0;
  bool ok = true;
  // a tile is two candidate blocks (128 key rows); virtual tile v walks (sequence, tile) pairs
  auto tiles_of = [&](int bb) { return (p.cnt[bb] + 1) / 2; };
  int b = 0, base_t = 0, nt_b = p.B > 0 ? tiles_of(0) : 0;
  for (int v = blockIdx.x; ok; v += gridDim.x) {
    while (b < p.B && v >= base_t + nt_b) {
      base_t += nt_b;
      ++b;
      nt_b = b < p.B ? tiles_of(b) : 0;
    }
    if (b >= p.B) break;
    const int tile = v - base_t;
    const int n_cand = p.cnt[b], n_b = p.sch.seq_len[b];
    if (b != cur_b) {  // this sequence's query (64 heads) and exact lse
      const __nv_bfloat16* q = p.qry + (size_t)b * H * D;
      for (int i = tid; i < H * D / 8; i += 128) {
        const int row = i / (D / 8), ch = i % (D / 8);
        cp_async_16(smem_u32(sQ) + (ch / 8) * (H * 128) + sw128_off(row, ch % 8), q + row * D + ch * 8, true);
      }
      if (tid < H) s_nl[tid] = -p.lse2x[b * H + tid];
      cur_b = b;
    }
    // row tid: token (candidate 2 * tile + tid / 64) * 64 + tid % 64, if it is at or before t
    const int slot = 2 * tile + (tid >> 6);
    const int blk_j = slot < n_cand ? p.cand[(size_t)b * p.max_blocks + slot] : -1;
    const long long j = blk_j >= 0 ? (long long)blk_j * 64 + (tid & 63) : -1;
    const bool valid = j >= 0 && j < n_b;
    const long long krow = valid ? (long long)b * p.N + j : -1;
    {
      const int sub = lane >> 4, ch = lane & 15;
#pragma unroll
      for (int it = 0; it < 16; ++it) {
        const int rr = 2 * it + sub;  // row within this warp's 32
        const long long kr = __shfl_sync(0xffffffffu, krow, rr);
        cp_async_16(smem_u32(sK) + (ch / 8) * (TILE * 128) + sw128_off(warp * 32 + rr, ch % 8),
                    p.kc + (size_t)(kr >= 0 ? kr : 0) * D + ch * 8, kr >= 0);
      }
    }
    cp_async_commit();
    cp_async_wait_all();
    fence_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t IDESC = idesc_bf16(TILE, H, 0, 0);
      const uint64_t ka = sdesc(smem_u32(sK), 16, 1024), qa = sdesc(smem_u32(sQ), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        umma_ss(tmem, sdesc_at(ka, (kk / 4) * (TILE * 128) + (kk % 4) * 32),
                sdesc_at(qa, (kk / 4) * (H * 128) + (kk % 4) * 32), IDESC, kk > 0);
      umma_commit(&mma_bar);
    }
    bool w_ok = true;
    if (tid == 0) w_ok = mbar_wait(&mma_bar, phase, p.wait_ns);
    if (!__syncthreads_and(w_ok)) { if (tid == 0) report_status(p.st, kStatusTimeout, 511); ok = false; break; }
    phase ^= 1;
    tc_fence_after();
    float sa = 0.f, sb = 0.f;
#pragma unroll
    for (int cc = 0; cc < H / 32; ++cc) {
      float sv[32];
      tmem_ld32(tmem + lane_base + cc * 32, sv);
      tmem_ld_wait();
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        float e0, e1;
        ffma2(e0, e1, sv[x], sv[x + 1], c, c, s_nl[cc * 32 + x], s_nl[cc * 32 + x + 1]);
        fadd2(sa, sb, sa, sb, fast_exp2(e0), fast_exp2(e1));
      }
    }
    // the block's sum: rows 0..63 are warps 0 and 1, rows 64..127 warps 2 and 3
    float s = valid ? sa + sb : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) wsum[warp] = s;
    tc_fence_before();
    __syncthreads();  // TMEM and the K tile are reused by the next tile; wsum is complete
    if (tid == 0) {
      float* out = p.bsc + (size_t)b * p.max_blocks;
      if (2 * tile < n_cand) out[2 * tile] = wsum[0] + wsum[1];
      if (2 * tile + 1 < n_cand) out[2 * tile + 1] = wsum[2] + wsum[3];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 64); }
}

__global__ void __launch_bounds__(NT) blk_final_kernel(BlkParams p) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int CHUNK = 2048, OWN = 8;
  __shared__ unsigned long long keys[CHUNK];
  __shared__ int s_sel[32];
  __shared__ int s_n;
  const int b = blockIdx.x, tid = threadIdx.x;
  const int n_b = p.sch.seq_len[b], t = n_b - 1;
  const int C = p.cnt[b];
  const int* cand = p.cand + (size_t)b * p.max_blocks;
  const float* bsc = p.bsc + (size_t)b * p.max_blocks;
  if (tid == 0) s_n = 0;
  __syncthreads();
  auto key_of = [&](int i) {  // larger key == higher score, then lower block
    return ((unsigned long long)__float_as_uint(bsc[i]) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)cand[i]);
  };
  if (C <= p.NB) {
    for (int i = tid; i < C; i += NT) s_sel[i] = cand[i];
    if (tid == 0) s_n = C;
  } else {
    // rank of each candidate = how many candidates have a larger key; the n_blocks of rank below
    // n_blocks are the chosen ones (keys are unique). Candidates i = tid + NT (g * OWN + x).
    for (int g0 = 0; g0 * NT * OWN < C; ++g0) {
      unsigned long long mine[OWN];
      int rank[OWN];
#pragma unroll
      for (int x = 0; x < OWN; ++x) {
        const int i = tid + NT * (g0 * OWN + x);
        mine[x] = i < C ? key_of(i) : 0ull;
        rank[x] = 0;
      }
      for (int c0 = 0; c0 < C; c0 += CHUNK) {
        const int n = C - c0 < CHUNK ? C - c0 : CHUNK;
        __syncthreads();
        for (int i = tid; i < n; i += NT) keys[i] = key_of(c0 + i);
        __syncthreads();
        for (int i = 0; i < n; ++i) {
          const unsigned long long kk = keys[i];
#pragma unroll
          for (int x = 0; x < OWN; ++x) rank[x] += kk > mine[x];
        }
      }
#pragma unroll
      for (int x = 0; x < OWN; ++x) {
        const int i = tid + NT * (g0 * OWN + x);
        if (i < C && rank[x] < p.NB) {
          const int at = atomicAdd(&s_n, 1);
          if (at < 32) s_sel[at] = cand[i];
        }
      }
    }
  }
  __syncthreads();
  const int n_sel = s_n < p.NB ? s_n : p.NB;
  if (tid == 0) {
    if (s_n != (C <= p.NB ? C : p.NB)) report_status(p.st, kStatusBounds, 521);
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
    LaunchScope ls("blk_bound", stream);
    const int per_seq = (p.H + NT / 32 - 1) / (NT / 32);
    e = launch_k(blk_bound_kernel, dim3(p.B + p.B * per_seq), dim3(NT), 0, stream, true, p);
  }
  if (e != cudaSuccess) return e;
  {
    static bool configured = false;
    constexpr int RS_SMEM = 1024 + 64 * 128 * 2 + 128 * 128 * 2;
    if (!configured) {
      cudaFuncSetAttribute(blk_rescore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RS_SMEM);
      configured = true;
    }
    int grid = 2 * (p.sms > 0 ? p.sms : 148);
    const int max_tiles = p.B * ((p.max_blocks + 1) / 2);
    if (grid > max_tiles) grid = max_tiles > 0 ? max_tiles : 1;
    LaunchScope ls("blk_rescore", stream);
    e = launch_k(blk_rescore_kernel, dim3(grid), dim3(128), RS_SMEM, stream, true, p);
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
