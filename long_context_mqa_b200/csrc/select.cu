// Exact top-k of the decode path, ties to the lower index, from the decode kernel's bounded
// scores (score' with score' / max L' <= score <= score' / min L', see decode.cu).
//
//  1. bounds   : (decode kernel, last CTA of a sequence) from the 2048-bin histogram of score'
//                bits 30..20: bins above b_hi hold keys certainly selected (`above` of them),
//                bins below b_lo keys certainly not; `need` = k - above are to come from the band
//                b_lo..b_hi.
//  2. collect  : every score' above b_hi sets its bit in the sequence's selection bitmap (one bit
//                per older token, cleared by the decode kernel); band keys are listed by index
//                (one list-counter update per warp).
//  3. rescore  : the band keys' K rows are gathered (an e4m3 cache's rows widened exactly to
//                bf16 on the way) and their exact scores computed (tcgen05, exact lse), as unique
//                64-bit keys (score bits << 32 | ~index: larger key == higher score, then lower
//                index).
//  4. final    : MSB-first 8-bit radix select of the `need` largest band keys (starting at the
//                highest bit on which they differ, stopping as soon as the chosen bucket holds
//                exactly the remaining need) sets their bits; one pass over the bitmap with a
//                block-wide prefix sum writes the chosen indices in ascending order, and the
//                forced window (every index of which is larger) is appended. Extra CTAs of the
//                same launch produce the decode output (independent of the selection): per
//                (sequence, head), the sum of the output records of the CTAs covering the
//                sequence, divided by L' (and multiplied by an e4m3 V cache's scale).
#include "combine.cuh"
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace sel {

constexpr int NT = 1024;

// The decode output of head h of sequence b, by one warp (lane = 4 columns).
__device__ __forceinline__ void combine_output(const SelParams& p, int b, int h, unsigned lane) {
  combine_decode_output(p.opart, p.lsum, p.oscale, p.out, p.H, p.D, p.sch, p.st, b, h, lane);
}

// Scores one bitmap CTA of the collect kernel classifies: 256 threads x 8 steps x 4 scores.
constexpr int COLLECT_CHUNK = 8192;

// Bitmap + band keys of scores [blockIdx.x * COLLECT_CHUNK, +COLLECT_CHUNK) of sequence blockIdx.y.
__global__ void __launch_bounds__(256) sel_collect_kernel(SelParams p) {
  griddep_wait();
  griddep_launch_dependents();
  // both decode launches are complete: re-arm their grid barrier for the next step
  if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *(volatile unsigned*)p.gbar = 0u;
  const int b = blockIdx.y;
  const unsigned lane = threadIdx.x & 31;
  int* meta = p.meta + b * META;
  const int beta = meta[0], beta_lo = meta[3];
  const float* sc = p.sc + (size_t)b * p.ncand;
  unsigned* bm = p.bitmap + (size_t)b * p.words;
  const int nc = p.sch.seq_len[b] - p.W > 0 ? p.sch.seq_len[b] - p.W : 0;  // this sequence's older tokens
  const bool vec = ((reinterpret_cast<uintptr_t>(sc) & 15u) == 0);
  const int c0 = blockIdx.x * COLLECT_CHUNK + threadIdx.x * 4;
  // four consecutive scores per thread per step (one bitmap word, one 16-byte load); the loads
  // of four steps are issued together. Band scores are marked in `band` (bit 4 * step + x) and
  // appended at the end with one counter update per warp.
  unsigned band = 0;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    float v[4][4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j0 = c0 + (half * 4 + k) * 1024;
      if (vec && j0 + 3 < nc) {
        const float4 f = __ldcg(reinterpret_cast<const float4*>(sc + j0));
        v[k][0] = f.x; v[k][1] = f.y; v[k][2] = f.z; v[k][3] = f.w;
      } else {
#pragma unroll
        for (int x = 0; x < 4; ++x) v[k][x] = j0 + x < nc ? __ldcg(sc + j0 + x) : 0.f;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j0 = c0 + (half * 4 + k) * 1024;
      unsigned upmask = 0;
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const int j = j0 + x;
        const bool in_range = j < nc;
        const uint32_t bits = __float_as_uint(v[k][x]);
        const int bin = in_range ? (int)((bits >> 20) & (NBINS - 1)) : -2;
        if (in_range && bin > beta) upmask |= 1u << (j & 31);
        if (in_range && bin >= beta_lo && bin <= beta) band |= 1u << ((half * 4 + k) * 4 + x);  // re-scored exactly
      }
      if (upmask) atomicOr(&bm[j0 >> 5], upmask);
    }
  }
  // the warp's band scores get consecutive slots of the sequence's band list
  const unsigned nb = __popc(band);
  unsigned incl = nb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= (unsigned)o) incl += n;
  }
  const unsigned total = __shfl_sync(0xffffffffu, incl, 31);
  if (total == 0) return;
  unsigned base = 0;
  if (lane == 31) base = (unsigned)atomicAdd(&meta[4], (int)total);
  unsigned pos = __shfl_sync(0xffffffffu, base, 31) + incl - nb;
  while (band) {
    const int bit = __ffs(band) - 1;
    band &= band - 1;
    const int j = c0 + (bit >> 2) * 1024 + (bit & 3);
    p.bnd[(size_t)b * p.ncand + pos++] = (unsigned long long)(uint32_t)j;
  }
}

__global__ void __launch_bounds__(128) sel_rescore_kernel(SelParams p) {
  griddep_wait();
  griddep_launch_dependents();
  constexpr int H = 64, D = 128, TILE = 128;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem;               // [64 heads][128] K-major SW128 (two 64-column blocks)
  uint8_t* sK = smem + H * D * 2;   // [128 keys][128] K-major SW128
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ __align__(16) float s_nl[H];  // -lse2 of the current sequence
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
  // virtual tile v walks (sequence, tile) pairs in sequence order; b, base_t follow it
  auto tiles_of = [&](int bb) { return (p.meta[bb * META + 4] + TILE - 1) / TILE; };
  int b = 0, base_t = 0, nt_b = p.B > 0 ? tiles_of(0) : 0;
  for (int v = blockIdx.x; ok; v += gridDim.x) {
    while (b < p.B && v >= base_t + nt_b) {
      base_t += nt_b;
      ++b;
      nt_b = b < p.B ? tiles_of(b) : 0;
    }
    if (b >= p.B) break;
    const int tile = v - base_t;
    const int n_band = p.meta[b * META + 4];
    if (b != cur_b) {  // this sequence's query (64 heads) and exact lse
      const __nv_bfloat16* q = p.qry + (size_t)b * H * D;
      for (int i = tid; i < H * D / 8; i += 128) {
        const int row = i / (D / 8), ch = i % (D / 8);
        cp_async_16(smem_u32(sQ) + (ch / 8) * (H * 128) + sw128_off(row, ch % 8), q + row * D + ch * 8, true);
      }
      if (tid < H) s_nl[tid] = -p.lse2x[b * H + tid];
      cur_b = b;
    }
    // gather the K rows of band slots tile*128 .. +127 (zero rows past the end). Thread `tid`
    // reads the index of row `tid`; the copies are coalesced, 16 lanes per row (the whole
    // 256-byte row), the row's index passed by shuffle
    const int slot = tile * TILE + tid;
    const bool in = slot < n_band;
    const int j = in ? (int)(uint32_t)p.bnd[(size_t)b * p.ncand + slot] : 0;
    bool valid = in && j >= 0 && j < p.sch.seq_len[b] - p.W;
    // the K row of key j: row j of sequence b's cache, or (paged) row j % 128 of its page
    long long krow = -1;
    if (valid) {
      if (p.ptab) {
        const int pg = __ldg(p.ptab + (size_t)b * p.max_pages + (j >> 7));
        if (pg >= 0 && pg < p.n_pages) krow = (long long)pg * 128 + (j & 127);
        else { valid = false; report_status(p.st, kStatusBounds, 313); }
      } else {
        krow = (long long)b * p.N + j;
      }
    }
    if (p.kc8) {
      // e4m3 cache: 128-byte rows, 8 lanes per row, 16 codes per lane widened exactly to bf16
      const int sub = lane >> 3, ch = lane & 7;
      uint4 x[8];
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const long long kr = __shfl_sync(0xffffffffu, krow, 4 * it + sub);
        x[it] = kr >= 0 ? __ldg(reinterpret_cast<const uint4*>(p.kc8 + (size_t)kr * D) + ch) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const uint32_t row_base = smem_u32(sK) + (ch / 4) * (TILE * 128);
        const int rr = warp * 32 + 4 * it + sub;
        st_shared_v4(row_base + sw128_off(rr, (2 * ch) % 8), e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].x)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].x >> 16)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].y)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].y >> 16)));
        st_shared_v4(row_base + sw128_off(rr, (2 * ch + 1) % 8), e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].z)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].z >> 16)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].w)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x[it].w >> 16)));
      }
    } else {
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
    if (!__syncthreads_and(w_ok)) { if (tid == 0) report_status(p.st, kStatusTimeout, 311); ok = false; break; }
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
    if (in && !valid) report_status(p.st, kStatusBounds, 312);
    if (in) {
      const float score = sa + sb;
      p.bnd[(size_t)b * p.ncand + slot] =
          ((unsigned long long)__float_as_uint(score) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)j);
    }
    tc_fence_before();
    __syncthreads();  // TMEM and the K tile are reused by the next tile
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 64); }
}

__global__ void __launch_bounds__(NT) sel_final_kernel(SelParams p) {
  griddep_wait();
  griddep_launch_dependents();
  if ((int)blockIdx.x >= p.B) {
    // the decode output (independent of the selection), a warp per head: NT / 32 heads per CTA
    const int oc = blockIdx.x - p.B, per_seq = (p.H + NT / 32 - 1) / (NT / 32);
    const int h = (oc % per_seq) * (NT / 32) + (int)(threadIdx.x >> 5);
    if (h < p.H) combine_output(p, oc / per_seq, h, threadIdx.x & 31);
    return;
  }
  constexpr int KPT = 4;  // band keys held in registers per thread (bands up to NT * KPT keys)
  constexpr int WPT = 8;  // bitmap words per thread per round of the ordered write-out
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  __shared__ unsigned dh[256];
  __shared__ unsigned long long s_prefix, s_mask, s_and, s_or;
  __shared__ int s_need, s_exact;
  __shared__ unsigned wsum[32];
  const int* meta = p.meta + b * META;
  const int need = meta[2];
  const int n_bnd = meta[4];
  const unsigned long long* bnd = p.bnd + (size_t)b * p.ncand;
  unsigned* bm = p.bitmap + (size_t)b * p.words;
  if (need > 0 && n_bnd > 0) {
    // the band keys, read once into registers when they fit (else every pass reads them again)
    const bool in_regs = n_bnd <= NT * KPT;
    unsigned long long kr[KPT];
#pragma unroll
    for (int x = 0; x < KPT; ++x) kr[x] = in_regs && tid + x * NT < n_bnd ? bnd[tid + x * NT] : 0ull;
    auto visit = [&](auto&& f) {
      if (in_regs) {
#pragma unroll
        for (int x = 0; x < KPT; ++x)
          if (tid + x * NT < n_bnd) f(kr[x]);
      } else {
        for (int i = tid; i < n_bnd; i += NT) f(bnd[i]);
      }
    };
    // bits on which every boundary key agrees need no pass: start at the highest differing bit
    if (tid == 0) { s_and = ~0ull; s_or = 0ull; s_need = need; s_exact = 0; }
    __syncthreads();
    unsigned long long a_loc = ~0ull, o_loc = 0ull;
    visit([&](unsigned long long key) { a_loc &= key; o_loc |= key; });
    for (int o = 16; o > 0; o >>= 1) {
      a_loc &= __shfl_xor_sync(0xffffffffu, a_loc, o);
      o_loc |= __shfl_xor_sync(0xffffffffu, o_loc, o);
    }
    if (lane == 0) { atomicAnd(&s_and, a_loc); atomicOr(&s_or, o_loc); }
    __syncthreads();
    const unsigned long long diff = s_and ^ s_or;
    const int top = diff ? 63 - __clzll((long long)diff) : 0;
    if (tid == 0) {
      s_mask = top >= 63 ? 0ull : ~((2ull << top) - 1ull);
      s_prefix = s_and & s_mask;
    }
    __syncthreads();
    // 8-bit digit windows from the top down; the last is clamped at bit 0 (its bits above the
    // previous window are already fixed in the prefix)
    for (int sh_raw = top - 7;; sh_raw -= 8) {
      const int shift = sh_raw < 0 ? 0 : sh_raw;
      for (int i = tid; i < 256; i += NT) dh[i] = 0;
      __syncthreads();
      const unsigned long long prefix = s_prefix, mask = s_mask;
      visit([&](unsigned long long key) {
        if ((key & mask) == prefix) atomicAdd(&dh[(key >> shift) & 255u], 1u);
      });
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
      if (shift == 0 || s_exact) break;
    }
    // keys whose masked prefix is >= s_prefix are exactly the `need` largest boundary entries
    const unsigned long long thr = s_prefix, fmask = s_mask;
    visit([&](unsigned long long key) {
      if ((key & fmask) >= thr) {
        const uint32_t j = 0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull);
        atomicOr(&bm[j >> 5], 1u << (j & 31));
      }
    });
  }
  __syncthreads();
  // the bitmap in order, in rounds of NT * WPT words: each thread owns WPT consecutive words
  // (two 16-byte loads: the bitmap's row stride is a multiple of 8 words), a block-wide
  // exclusive scan of their counts gives its output position
  int32_t* out = p.idx + (size_t)b * p.S;
  unsigned done = 0;  // chosen indices written in earlier rounds
  for (int base = 0; base < p.words; base += NT * WPT) {
    const int w0 = base + tid * WPT;
    unsigned wv[WPT], cnt = 0;
    if (w0 < p.words) {
      const uint4 a = __ldcg(reinterpret_cast<const uint4*>(bm + w0));
      const uint4 c4 = __ldcg(reinterpret_cast<const uint4*>(bm + w0 + 4));
      wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w; wv[4] = c4.x; wv[5] = c4.y; wv[6] = c4.z; wv[7] = c4.w;
    } else {
#pragma unroll
      for (int x = 0; x < WPT; ++x) wv[x] = 0u;
    }
#pragma unroll
    for (int x = 0; x < WPT; ++x) cnt += __popc(wv[x]);
    unsigned incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned n = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += n;
    }
    if (lane == 31) wsum[w] = incl;
    __syncthreads();
    if (w == 0) {
      unsigned t = wsum[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned n = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += n;
      }
      wsum[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    unsigned pos = done + incl - cnt + (w > 0 ? wsum[w - 1] : 0u);
#pragma unroll
    for (int x = 0; x < WPT; ++x) {
      unsigned word = wv[x];
      while (word) {
        const int bit = __ffs(word) - 1;
        word &= word - 1;
        if (pos < (unsigned)p.S) out[pos] = (w0 + x) * 32 + bit;
        ++pos;
      }
    }
    done += wsum[31];
    __syncthreads();  // wsum is rewritten by the next round
  }
  const unsigned total_top = done;
  const int n_b = p.sch.seq_len[b], nc = n_b - p.W > 0 ? n_b - p.W : 0;  // this sequence's
  const int wlen = n_b < p.W ? n_b : p.W;
  const int expect_top = nc < p.K ? nc : p.K;
  if (tid == 0 && (int)total_top != expect_top) report_status(p.st, kStatusBounds, 302);
  for (int i = tid; i < p.S; i += NT) {
    if (i >= (int)total_top && i < (int)total_top + wlen) out[i] = n_b - wlen + (i - (int)total_top);
    else if (i >= (int)total_top + wlen) out[i] = -1;
  }
}

cudaError_t launch_select(const SelParams& p, cudaStream_t stream) {
  cudaError_t e;
  {
    int n_collect = (p.ncand + COLLECT_CHUNK - 1) / COLLECT_CHUNK;
    if (n_collect < 1) n_collect = 1;
    LaunchScope ls("sel_collect", stream);
    e = launch_k(sel_collect_kernel, dim3(n_collect, p.B), dim3(256), 0, stream, true, p);
  }
  if (e != cudaSuccess) return e;
  {
    static bool configured = false;
    constexpr int RS_SMEM = 1024 + 64 * 128 * 2 + 128 * 128 * 2;
    if (!configured) {
      cudaFuncSetAttribute(sel_rescore_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, RS_SMEM);
      configured = true;
    }
    int grid = 2 * (p.sms > 0 ? p.sms : 148);
    const int max_tiles = p.B * ((p.ncand + 127) / 128);
    if (grid > max_tiles) grid = max_tiles > 0 ? max_tiles : 1;
    LaunchScope ls("sel_rescore", stream);
    e = launch_k(sel_rescore_kernel, dim3(grid), dim3(128), RS_SMEM, stream, true, p);
  }
  if (e != cudaSuccess) return e;
  {
    LaunchScope ls("sel_final", stream);
    // B selection CTAs, then the output CTAs
    const int per_seq = (p.H + NT / 32 - 1) / (NT / 32);
    e = launch_k(sel_final_kernel, dim3(p.B + p.B * per_seq), dim3(NT), 0, stream, true, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace sel
}  // namespace hs2
