// Prefill full attention + token selection: Lq queries at positions off + 0 .. off + Lq - 1
// (off = Lk - Lq: Lq == Lk is a whole prompt, Lq < Lk a chunk appended to a cache).
//
// Pass 1, fa_fwd: causal MQA flash attention producing out and the per-(query, head) logsumexp.
//   Rows of a 128-row tile are (query, head) pairs -- all heads of 128/H consecutive queries --
//   so one K/V tile of the single KV head serves every head (MQA). One work item = two such
//   tiles (A and B), each owned by one softmax warpgroup; the tcgen05 issuer ping-pongs
//   S_A = Q_A K^T, S_B = Q_B K^T, O_A += P_A V, O_B += P_B V so the tensor core stays busy while
//   either warpgroup does its softmax. S and O live in TMEM (4 x 128 columns); P (bf16) is
//   staged K-major in shared memory; K and V tiles stream through a 3-slot TMA ring. The
//   running row max is raised lazily (only when a tile exceeds it by more than 2^8), and only
//   then is the thread's O row rescaled in TMEM.
//
// Pass 2, score_select: the exact head-summed probabilities and the top-k choice, without ever
//   materialising the L x L matrix. Tiles are transposed -- S^T = K_tile Q_item^T with 128 keys in
//   TMEM lanes and N = 256 (query, head) columns -- so the sum over heads is an in-thread
//   reduction: score(t, j) = sum_h exp2(s * c - lse2(t, h)) with pass 1's lse. Every query keeps a
//   candidate buffer in shared memory of unique 64-bit keys (score bits << 32 | ~index: larger key
//   == higher score, then lower index). A key enters only if it beats the query's current
//   threshold; when the buffer nears capacity an exact MSB radix select keeps the top-k and
//   raises the threshold. Keys are visited newest first. At the end the kept indices are
//   written ascending (a bitmap over the candidate range and one prefix count; a sort only past
//   the bitmap's capacity), then the forced window.
//
// Both kernels are persistent: CTAs take work items in order of decreasing causal work, round
// robin. Warp roles: warp 0 TMA producer, warp 1 tcgen05 issuer + TMEM owner, then the softmax
// warpgroups (warp w reads TMEM lanes 32*(w%4)..+31): fa_fwd (320 threads) warps 2..5 and 6..9
// for tiles A and B; score_select (576 threads) four warpgroups, each owning a quarter of the 256
// (query, head) columns, i.e. a quarter of the item's queries. Every wait is bounded and reports
// a timeout through the status word.
#include "decode.h"
#include "host_util.h"
#include "prefill.h"
#include "tc.cuh"

namespace hs2 {
namespace prefill {

constexpr int NT = 320;
constexpr int SC_WG = 4;                 // score pass: softmax warpgroups
constexpr int NT_SC = 64 + 128 * SC_WG;  // score pass: + the producer and issuer warps
constexpr float LOG2E = 1.4426950408889634f;
// Of every 16 score-pass exponentials, how many exp2_fma2 computes on the FMA pipes instead of
// the MUFU. Measured on B200 at L = 32k with four softmax warpgroups: 0, 4 and 6 give 12.96, 12.95
// and 13.51 ms, so the MUFU does all of them.
constexpr int SOFT_EXP2 = 0;

struct PfParams {
  int B, Lq, Lk, H;
  int off;              // Lk - Lq: query i sits at position off + i
  int rows_per_batch;   // Lq * H
  int items_per_batch;  // ceil(Lq * H / 256)
  int n_items;
  float c;              // scale * log2(e)
  int W, K, S;
  __nv_bfloat16* out;
  float* lse;
  int32_t* idx;
  long long wait_ns;
  DevStatus* st;
};

__device__ __forceinline__ bool wait_abortable(uint64_t* bar, uint32_t parity, long long limit, volatile int* abort_flag,
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
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, long long limit, volatile int* abort_flag,
                                          DevStatus* st, unsigned where) {
  if (__all_sync(0xffffffffu, mbar_try_wait(smem_u32(bar), parity))) return true;  // completed: no divergent wait
  int ok = 1;
  if ((threadIdx.x & 31) == 0) ok = wait_abortable(bar, parity, limit, abort_flag, st, where) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}
__device__ __forceinline__ void wg_bar(int wg) {  // named barrier of one 128-thread warpgroup
  asm volatile("bar.sync %0, 128;" ::"r"(1 + wg) : "memory");
}

// =============================================================================================
// pass 1: flash attention forward
// =============================================================================================
template <int H, int D>
struct FaCfg {
  static constexpr int QPT = 128 / H;
  static constexpr int Q_BYTES = 128 * D * 2;
  static constexpr int KV_BYTES = 128 * D * 2;
  static constexpr int P_BYTES = 128 * 128 * 2;
  static constexpr int RING = 3;
  static constexpr int OFF_Q = 0;                       // Q_A, Q_B
  static constexpr int OFF_P = 2 * Q_BYTES;             // P_A, P_B
  static constexpr int OFF_RING = OFF_P + 2 * P_BYTES;
  static constexpr int SMEM = 1024 + OFF_RING + RING * KV_BYTES;
};

// key tiles an item covers: 0 .. last_tile
__device__ __forceinline__ int fa_last_tile(const PfParams& p, int item_in_batch) {
  int t_hi = (item_in_batch * 256 + 255) / p.H;
  if (t_hi > p.Lq - 1) t_hi = p.Lq - 1;
  return (p.off + t_hi) / 128;
}

template <int H, int D>
__global__ void __launch_bounds__(NT, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, PfParams p) {
  using C = FaCfg<H, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t q_full, q_empty, r_full[C::RING], r_empty[C::RING], s_full[2], s_empty[2],
      p_full[2], pv_done[2];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const long long limit = p.wait_ns;
  const uint32_t tS = 0, tO = 256;  // S_w at tS + 128 w, O_w at tO + D w

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int i = 0; i < C::RING; ++i) { mbar_init(&r_full[i], 1); mbar_init(&r_empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 4);
      mbar_init(&p_full[i], 4); mbar_init(&pv_done[i], 1);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
      uint32_t ri = 0;
      int it = 0;
      bool ok = true;
      for (int item = p.n_items - 1 - blockIdx.x; item >= 0 && ok; item -= gridDim.x, ++it) {
        const int b = item / p.items_per_batch, ib = item % p.items_per_batch;
        const int r0 = b * p.rows_per_batch + ib * 256;
        const int jt = fa_last_tile(p, ib);
        if (!wait_abortable(&q_empty, (it & 1) ^ 1, limit, &abort_flag, p.st, 601)) { ok = false; break; }
        mbar_expect_tx(&q_full, 2 * C::Q_BYTES);
        for (int w = 0; w < 2; ++w)
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_2d(smem + C::OFF_Q + w * C::Q_BYTES + kb * (128 * 128), &tmQ, &q_full, kb * 64, r0 + w * 128);
        for (int j = 0; j <= jt && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++ri) {
            const int s = ri % C::RING;
            if (!wait_abortable(&r_empty[s], ((ri / C::RING) & 1) ^ 1, limit, &abort_flag, p.st, 602)) { ok = false; break; }
            mbar_expect_tx(&r_full[s], C::KV_BYTES);
            uint8_t* dst = smem + C::OFF_RING + s * C::KV_BYTES;
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(dst + kb * (128 * 128), kv == 0 ? &tmK : &tmV, &r_full[s], kb * 64, j * 128, b);
          }
        }
      }
      if (!ok)
        for (uint32_t x = (ri > C::RING ? ri - C::RING : 0); x < ri; ++x)
          mbar_wait(&r_full[x % C::RING], (x / C::RING) & 1, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t IDESC_O = idesc_bf16(128, D, 0, 1);
      uint32_t ri = 0;            // ring index of the next K tile
      uint32_t ns[2] = {0, 0};    // S issues per warpgroup
      uint32_t npv[2] = {0, 0};   // PV issues per warpgroup
      int it = 0;
      bool ok = true;
      auto issue_s = [&](int w, uint32_t kslot_idx) -> bool {
        const int s = kslot_idx % C::RING;
        if (!wait_abortable(&r_full[s], (kslot_idx / C::RING) & 1, limit, &abort_flag, p.st, 611)) return false;
        if (!wait_abortable(&s_empty[w], (ns[w] & 1) ^ 1, limit, &abort_flag, p.st, 612)) return false;
        tc_fence_after();
        const uint64_t qa = sdesc(smem_u32(smem + C::OFF_Q + w * C::Q_BYTES), 16, 1024);
        const uint64_t ka = sdesc(smem_u32(smem + C::OFF_RING + s * C::KV_BYTES), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sdesc_at(qa, (kk / 4) * (128 * 128) + (kk % 4) * 32);
          const uint64_t bk = sdesc_at(ka, (kk / 4) * (128 * 128) + (kk % 4) * 32);
          umma_ss(tmem + tS + 128 * w, a, bk, IDESC_S, kk > 0);
        }
        umma_commit(&s_full[w]);
        ns[w]++;
        return true;
      };
      auto issue_pv = [&](int w, uint32_t vslot_idx, bool first) -> bool {
        const int s = vslot_idx % C::RING;
        if (!wait_abortable(&p_full[w], npv[w] & 1, limit, &abort_flag, p.st, 613)) return false;
        if (!wait_abortable(&r_full[s], (vslot_idx / C::RING) & 1, limit, &abort_flag, p.st, 614)) return false;
        tc_fence_after();
        const uint64_t pa = sdesc(smem_u32(smem + C::OFF_P + w * C::P_BYTES), 16, 1024);
        const uint64_t va = sdesc(smem_u32(smem + C::OFF_RING + s * C::KV_BYTES), 128 * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          const uint64_t a = sdesc_at(pa, (kk / 4) * (128 * 128) + (kk % 4) * 32);
          const uint64_t bv = sdesc_at(va, kk * 2048);
          umma_ss(tmem + tO + D * w, a, bv, IDESC_O, (first && kk == 0) ? 0u : 1u);
        }
        umma_commit(&pv_done[w]);
        npv[w]++;
        return true;
      };
      for (int item = p.n_items - 1 - blockIdx.x; item >= 0 && ok; item -= gridDim.x, ++it) {
        const int ib = item % p.items_per_batch;
        const int jt = fa_last_tile(p, ib);
        if (!wait_abortable(&q_full, it & 1, limit, &abort_flag, p.st, 610)) { ok = false; break; }
        const uint32_t base = ri;  // K_j at base + 2j, V_j at base + 2j + 1
        if (!issue_s(0, base) || !issue_s(1, base)) { ok = false; break; }
        umma_commit(&r_empty[base % C::RING]);  // K_0 consumed
        for (int j = 0; j <= jt; ++j) {
          const uint32_t kj1 = base + 2 * (j + 1), vj = base + 2 * j + 1;
          if (!issue_pv(0, vj, j == 0)) { ok = false; break; }
          if (j < jt && !issue_s(0, kj1)) { ok = false; break; }
          if (!issue_pv(1, vj, j == 0)) { ok = false; break; }
          umma_commit(&r_empty[vj % C::RING]);  // V_j consumed
          if (j < jt) {
            if (!issue_s(1, kj1)) { ok = false; break; }
            umma_commit(&r_empty[kj1 % C::RING]);  // K_{j+1} consumed
          }
        }
        if (!ok) break;
        umma_commit(&q_empty);
        ri = base + 2 * (jt + 1);
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax warpgroups
    const int w = (warp - 2) / 4;       // 0: tile A, 1: tile B
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t sS = tmem + lane_base + tS + 128 * w;
    const uint32_t sO = tmem + lane_base + tO + D * w;
    const uint32_t pbase = smem_u32(smem + C::OFF_P + w * C::P_BYTES);
    const float c = p.c;
    uint32_t n_s = 0, n_pv = 0;
    bool ok = true;
    for (int item = p.n_items - 1 - blockIdx.x; item >= 0 && ok; item -= gridDim.x) {
      const int b = item / p.items_per_batch, ib = item % p.items_per_batch;
      const int jt = fa_last_tile(p, ib);
      const int rloc = ib * 256 + w * 128 + row;      // row within the batch
      const bool valid_row = rloc < p.rows_per_batch;
      const int t = p.off + rloc / H;  // the row's query position
      float m_used = -INFINITY, l = 0.f;
      for (int j = 0; j <= jt; ++j) {
        if (!warp_wait(&s_full[w], n_s & 1, limit, &abort_flag, p.st, 621)) { ok = false; break; }
        n_s++;
        tc_fence_after();
        // causal masking only where the tile reaches past some row's query (warp-uniform)
        const bool masked = __any_sync(0xffffffffu, j * 128 + 127 > t);
        const int kvis = t - j * 128;  // keys 0..kvis of this tile are visible to this row
        // pass over S: max of the raw logits (c > 0, so scaling commutes with the max), 64 columns
        // per TMEM wait
        float rmax = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v[2][32];
          tmem_ld32(sS + hh * 64, v[0]);
          tmem_ld32(sS + hh * 64 + 32, v[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int cc = 2 * hh + c2;
            if (masked) {
#pragma unroll
              for (int x = 0; x < 32; ++x) v[c2][x] = cc * 32 + x <= kvis ? v[c2][x] : -INFINITY;
            }
            rmax = fmaxf(rmax, max32(v[c2]));
          }
        }
        const float mx = rmax * c;
        const bool raise = mx > -INFINITY && (m_used == -INFINITY || mx > m_used + 8.f);
        const float m_new = raise ? mx : m_used;
        const float alpha = raise ? (m_used == -INFINITY ? 0.f : fast_exp2(m_used - m_new)) : 1.f;
        // P buffer and O of this warpgroup are free once the previous PV finished
        if (j > 0) {
          if (!warp_wait(&pv_done[w], n_pv & 1, limit, &abort_flag, p.st, 622)) { ok = false; break; }
          n_pv++;
          tc_fence_after();
          if (__any_sync(0xffffffffu, raise)) {
#pragma unroll
            for (int cc = 0; cc < D / 16; ++cc) {
              float o[16];
              tmem_ld16(sO + cc * 16, o);
              tmem_ld_wait();
#pragma unroll
              for (int x = 0; x < 16; ++x) o[x] *= alpha;
              tmem_st16(sO + cc * 16, o);
            }
            tmem_st_wait();
          }
        }
        l *= alpha;
        m_used = m_new;
        const float negm = -m_used;
        // probabilities -> P (K-major: row = this thread's (query, head), K = the 128 keys)
        float la = 0.f, lb = 0.f;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float vv[2][32];
          tmem_ld32(sS + hh * 64, vv[0]);
          tmem_ld32(sS + hh * 64 + 32, vv[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
          const int cc = 2 * hh + c2;
          const float* v = vv[c2];
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float e0, e1;
            ffma2(e0, e1, v[x], v[x + 1], c, c, negm, negm);
            float p0 = fast_exp2(e0), p1 = fast_exp2(e1);
            if (masked) {
              p0 = cc * 32 + x <= kvis ? p0 : 0.f;
              p1 = cc * 32 + x + 1 <= kvis ? p1 : 0.f;
            }
            fadd2(la, lb, la, lb, p0, p1);
            pk[x / 2] = pack_bf16x2(p0, p1);
          }
          const uint32_t blk = pbase + (cc / 2) * (128 * 128);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(blk + sw128_off(row, (cc % 2) * 4 + q), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
          }
        }
        l += la + lb;
        tc_fence_before();
        fence_async_smem();
        __syncwarp();
        if (lane == 0) { mbar_arrive(&s_empty[w]); mbar_arrive(&p_full[w]); }
      }
      if (!ok) break;
      // epilogue: O / l
      if (!warp_wait(&pv_done[w], n_pv & 1, limit, &abort_flag, p.st, 623)) { ok = false; break; }
      n_pv++;
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      __nv_bfloat16* orow = p.out + ((size_t)b * p.rows_per_batch + rloc) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        tmem_ld32(sO + cc * 32, o);
        tmem_ld_wait();
        if (valid_row) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(o[2 * x] * inv, o[2 * x + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
      if (valid_row) p.lse[(size_t)b * p.rows_per_batch + rloc] = (m_used + __log2f(l)) * 0.69314718055994531f;
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// =============================================================================================
// pass 2: head-summed scores + exact top-k per query
// =============================================================================================
template <int H, int D>
struct ScCfg {
  static constexpr int NQ = 256 / H;        // queries per item
  static constexpr int QW = NQ / SC_WG;     // queries per warpgroup
  static constexpr int CW = 256 / SC_WG;    // S columns per warpgroup (QW queries x H heads)
  static constexpr int CAP = H == 64 ? 1920 : 1152;  // candidate slots per query
  static constexpr int Q_BYTES = 256 * D * 2;
  static constexpr int KT_BYTES = 128 * D * 2;
  static constexpr int KST = H == 64 ? 3 : 2;        // K tiles in flight (from L2)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = Q_BYTES;
  static constexpr int OFF_C = OFF_K + KST * KT_BYTES;
  static constexpr int SMEM = 1024 + OFF_C + NQ * CAP * 8;
};

struct ScItem {
  int b, ib, tq0, t_hi, n_tiles;
};
__device__ __forceinline__ ScItem sc_item(const PfParams& p, int item, int nq) {
  ScItem s;
  s.b = item / p.items_per_batch;
  s.ib = item % p.items_per_batch;
  s.tq0 = s.ib * nq;
  s.t_hi = s.tq0 + nq - 1 < p.Lq - 1 ? s.tq0 + nq - 1 : p.Lq - 1;
  const int last_cand = p.off + s.t_hi - p.W;  // the newest older key of the item's last query
  s.n_tiles = last_cand >= 0 ? last_cand / 128 + 1 : 0;
  return s;
}

// Keeps the `keep` largest of the n unique keys in buf (WG-cooperative, 128 threads); returns the
// smallest kept key (the new admission threshold). n <= CAP.
template <int CAP>
__device__ unsigned long long wg_compact(unsigned long long* buf, int n, int keep, int wg, int wt, unsigned* hist,
                                         unsigned long long* s_prefix, int* s_need, int* s_cnt) {
  // bits on which all n keys agree need no radix pass: find the highest differing bit first
  __shared__ unsigned long long s_and[SC_WG], s_or[SC_WG];
  __shared__ int s_exact[SC_WG];
  if (wt == 0) { s_and[wg] = ~0ull; s_or[wg] = 0ull; *s_need = keep; *s_cnt = 0; s_exact[wg] = 0; }
  wg_bar(wg);
  {
    unsigned long long a = ~0ull, o = 0ull;
    for (int i = wt; i < n; i += 128) { const unsigned long long key = buf[i]; a &= key; o |= key; }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      a &= __shfl_xor_sync(0xffffffffu, a, off);
      o |= __shfl_xor_sync(0xffffffffu, o, off);
    }
    if ((wt & 31) == 0) { atomicAnd(&s_and[wg], a); atomicOr(&s_or[wg], o); }
  }
  wg_bar(wg);
  const unsigned long long diff = s_and[wg] ^ s_or[wg];
  const int top = diff ? 63 - __clzll((long long)diff) : 0;
  unsigned long long mask = top >= 63 ? 0ull : ~((2ull << top) - 1ull);
  if (wt == 0) *s_prefix = s_and[wg] & mask;
  wg_bar(wg);
  // 8-bit digit windows from the highest differing bit down; the last is clamped at bit 0
  for (int sh_raw = top - 7;; sh_raw -= 8) {
    const int shift = sh_raw < 0 ? 0 : sh_raw;
    for (int i = wt; i < 256; i += 128) hist[i] = 0u;
    wg_bar(wg);
    const unsigned long long prefix = *s_prefix;
    for (int i = wt; i < n; i += 128) {
      const unsigned long long key = buf[i];
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    wg_bar(wg);
    if (wt < 32) {
      const int ln = wt;
      unsigned cnt[8], tot = 0;
#pragma unroll
      for (int x = 0; x < 8; ++x) { cnt[x] = hist[255 - 8 * ln - x]; tot += cnt[x]; }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned v = __shfl_up_sync(0xffffffffu, incl, o);
        if (ln >= o) incl += v;
      }
      const unsigned excl = incl - tot;
      const unsigned k = (unsigned)*s_need;
      if (excl < k && incl >= k) {
        unsigned run = excl;
        for (int x = 0; x < 8; ++x) {
          if (run + cnt[x] >= k) {
            *s_need = (int)(k - run);
            *s_prefix = prefix | ((unsigned long long)(255u - 8u * ln - x) << shift);
            s_exact[wg] = run + cnt[x] == k;  // the whole bucket is kept: no further digit needed
            break;
          }
          run += cnt[x];
        }
      }
    }
    mask |= 255ull << shift;
    wg_bar(wg);
    if (shift == 0 || s_exact[wg]) break;
  }
  // keys whose masked prefix is >= the chosen prefix are exactly the `keep` largest
  const unsigned long long thr = *s_prefix;
  constexpr int PER = CAP / 128;
  unsigned long long mine[PER];
  int nm = 0;
#pragma unroll
  for (int m = 0; m < PER; ++m) {
    const int i = wt + 128 * m;
    mine[m] = 0ull;
    if (i < n) {
      const unsigned long long key = buf[i];
      if ((key & mask) >= thr) { mine[m] = key; nm++; }
    }
  }
  wg_bar(wg);
  int pos = nm ? atomicAdd(s_cnt, nm) : 0;
#pragma unroll
  for (int m = 0; m < PER; ++m)
    if (mine[m] != 0ull) buf[pos++] = mine[m];
  wg_bar(wg);
  return thr;
}

template <int H, int D>
__global__ void __launch_bounds__(NT_SC, 1)
    score_select_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK, PfParams p) {
  using C = ScCfg<H, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned long long* cbuf = reinterpret_cast<unsigned long long*>(smem + C::OFF_C);
  __shared__ __align__(8) uint64_t q_full, q_empty, k_full[C::KST], k_empty[C::KST], s_full[2], s_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  __shared__ __align__(16) float slse2[256];
  __shared__ int cnt[C::NQ];
  __shared__ unsigned long long theta[C::NQ];
  __shared__ unsigned hist[SC_WG][256];
  __shared__ unsigned long long s_prefix[SC_WG];
  __shared__ int s_need[SC_WG], s_cnt[SC_WG];
  __shared__ unsigned s_wsum[SC_WG][4];  // per-warp totals of the final ordered write
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const long long limit = p.wait_ns;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    mbar_init(&q_empty, 1);
    for (int i = 0; i < C::KST; ++i) { mbar_init(&k_full[i], 1); mbar_init(&k_empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&s_full[i], 1); mbar_init(&s_empty[i], 4 * SC_WG); }
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmK);
      uint32_t kt = 0;
      int it = 0;
      bool ok = true;
      for (int item = p.n_items - 1 - blockIdx.x; item >= 0 && ok; item -= gridDim.x) {
        const ScItem si = sc_item(p, item, C::NQ);
        if (si.n_tiles == 0) continue;
        if (!wait_abortable(&q_empty, (it & 1) ^ 1, limit, &abort_flag, p.st, 701)) { ok = false; break; }
        const int r0 = si.b * p.rows_per_batch + si.ib * 256;
        mbar_expect_tx(&q_full, C::Q_BYTES);
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(smem + C::OFF_Q + kb * (256 * 128), &tmQ, &q_full, kb * 64, r0);
        ++it;
        for (int j = si.n_tiles - 1; j >= 0; --j, ++kt) {
          const int s = kt % C::KST;
          if (!wait_abortable(&k_empty[s], ((kt / C::KST) & 1) ^ 1, limit, &abort_flag, p.st, 702)) { ok = false; break; }
          mbar_expect_tx(&k_full[s], C::KT_BYTES);
          for (int kb = 0; kb < D / 64; ++kb)
            tma_load_3d(smem + C::OFF_K + s * C::KT_BYTES + kb * (128 * 128), &tmK, &k_full[s], kb * 64, j * 128, si.b);
        }
      }
      if (!ok)
        for (uint32_t x = (kt > C::KST ? kt - C::KST : 0); x < kt; ++x)
          mbar_wait(&k_full[x % C::KST], (x / C::KST) & 1, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(128, 256, 0, 0);
      uint32_t kt = 0;
      int it = 0;
      bool ok = true;
      for (int item = p.n_items - 1 - blockIdx.x; item >= 0 && ok; item -= gridDim.x) {
        const ScItem si = sc_item(p, item, C::NQ);
        if (si.n_tiles == 0) continue;
        if (!wait_abortable(&q_full, it & 1, limit, &abort_flag, p.st, 711)) { ok = false; break; }
        ++it;
        const uint64_t qd = sdesc(smem_u32(smem + C::OFF_Q), 16, 1024);
        for (int j = si.n_tiles - 1; j >= 0; --j, ++kt) {
          const int s = kt % C::KST, buf = kt & 1;
          if (!wait_abortable(&k_full[s], (kt / C::KST) & 1, limit, &abort_flag, p.st, 712)) { ok = false; break; }
          if (!wait_abortable(&s_empty[buf], ((kt >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 713)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ka = sdesc(smem_u32(smem + C::OFF_K + s * C::KT_BYTES), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sdesc_at(ka, (kk / 4) * (128 * 128) + (kk % 4) * 32);
            const uint64_t bq = sdesc_at(qd, (kk / 4) * (256 * 128) + (kk % 4) * 32);
            umma_ss(tmem + buf * 256, a, bq, IDESC, kk > 0);
          }
          umma_commit(&s_full[buf]);
          umma_commit(&k_empty[s]);
        }
        if (!ok) break;
        umma_commit(&q_empty);
      }
    }
  } else {
    const int wg = (warp - 2) / 4;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;   // key within the tile
    const int wt = (warp - 2) % 4 * 32 + lane;  // thread index within the warpgroup
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float c = p.c;
    const unsigned lt_mask = (1u << lane) - 1u;
    uint32_t kt = 0;
    bool ok = true;
    // after a failed wait every later wait returns at once: the loop and named-barrier
    // structure stays identical across the warpgroup, only the tile work is skipped
    for (int item = p.n_items - 1 - blockIdx.x; item >= 0; item -= gridDim.x) {
      const ScItem si = sc_item(p, item, C::NQ);
      // per-query state of this warpgroup's queries
      for (int q = wt; q < C::QW; q += 128) {
        cnt[wg * C::QW + q] = 0;
        theta[wg * C::QW + q] = 0ull;
      }
      for (int x = wt; x < C::QW * H; x += 128) {
        const int q = wg * C::QW + x / H, h = x % H;
        const int t = si.tq0 + q;
        const float l = t < p.Lq ? p.lse[((size_t)si.b * p.Lq + t) * H + h] : 0.f;
        slse2[q * H + h] = -l * LOG2E;  // stored negated: one FFMA gives s*c - lse2
      }
      wg_bar(wg);
      for (int j = si.n_tiles - 1; j >= 0; --j, ++kt) {
        const int buf = kt & 1;
        if (ok && !warp_wait(&s_full[buf], (kt >> 1) & 1, limit, &abort_flag, p.st, 721)) ok = false;
        if (ok) {
        tc_fence_after();
        const int key = j * 128 + row;
        // this warpgroup's 64 columns (QW queries x H heads) in one go: the TMEM load latency
        // is paid once per tile, not once per 16 columns
        static_assert(C::CW == 64, "two 32-column loads per tile");
        float v0[32], v1[32];
        tmem_ld32(tmem + lane_base + buf * 256 + wg * C::CW, v0);
        tmem_ld32(tmem + lane_base + buf * 256 + wg * C::CW + 32, v1);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[buf]);  // the S buffer is free for the next tile
        auto col = [&](int i) -> float { return i < 32 ? v0[i] : v1[i - 32]; };
#pragma unroll
        for (int qq = 0; qq < C::QW; ++qq) {
          const int q = wg * C::QW + qq;
          const int t = si.tq0 + q;
          const bool cand = t < p.Lq && key <= p.off + t - p.W;
          if (!__any_sync(0xffffffffu, cand)) continue;  // warp-uniform: no lane has a candidate here
          // the exponentials can be shared between the MUFU (ex2) and the FMA pipes (exp2_fma2);
          // four independent pairs of partial sums keep the additions off one dependency chain
          float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int hc = 0; hc < H; hc += 16) {
            float e[16];
#pragma unroll
            for (int x = 0; x < 16; x += 4) {
              const float4 nl = *reinterpret_cast<const float4*>(&slse2[q * H + hc + x]);  // -lse2
              const int i = qq * H + hc + x;
              ffma2(e[x], e[x + 1], col(i), col(i + 1), c, c, nl.x, nl.y);
              ffma2(e[x + 2], e[x + 3], col(i + 2), col(i + 3), c, c, nl.z, nl.w);
            }
#pragma unroll
            for (int x = 0; x < SOFT_EXP2; x += 2) exp2_fma2(e[x], e[x + 1]);
#pragma unroll
            for (int x = SOFT_EXP2; x < 16; ++x) e[x] = fast_exp2(e[x]);
#pragma unroll
            for (int x = 0; x < 16; x += 2) {
              const int a = (x / 2) % 4;
              fadd2(acc[2 * a], acc[2 * a + 1], acc[2 * a], acc[2 * a + 1], e[x], e[x + 1]);
            }
          }
          const float score = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          const unsigned long long k64 =
              ((unsigned long long)__float_as_uint(score) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)key);
          const bool take = cand && k64 > theta[q];
          const unsigned m = __ballot_sync(0xffffffffu, take);
          if (m) {
            int base = 0;
            const int leader = __ffs(m) - 1;
            if (lane == leader) base = atomicAdd(&cnt[q], __popc(m));
            base = __shfl_sync(0xffffffffu, base, leader);
            if (take) cbuf[(size_t)q * C::CAP + base + __popc(m & lt_mask)] = k64;
          }
        }
        }
        wg_bar(wg);
        for (int qq = 0; qq < C::QW; ++qq) {
          const int q = wg * C::QW + qq;
          if (cnt[q] > C::CAP - 128) {
            theta[q] = wg_compact<C::CAP>(cbuf + (size_t)q * C::CAP, cnt[q], p.K, wg, wt, hist[wg], &s_prefix[wg],
                                          &s_need[wg], &s_cnt[wg]);
            if (wt == 0) cnt[q] = p.K;
            wg_bar(wg);
          }
        }
      }
      // final: top-k of each query, plus the forced window, sorted ascending
      for (int qq = 0; qq < C::QW; ++qq) {
        const int q = wg * C::QW + qq;
        const int t = si.tq0 + q;
        if (t >= p.Lq) continue;  // uniform across the warpgroup
        const int pos = p.off + t;  // the query's position
        const int n = cnt[q];
        const int keep = n < p.K ? n : p.K;
        unsigned long long* qb = cbuf + (size_t)q * C::CAP;
        if (n > keep) wg_compact<C::CAP>(qb, n, keep, wg, wt, hist[wg], &s_prefix[wg], &s_need[wg], &s_cnt[wg]);
        // keys -> indices (registers first, then overwrite the buffer as int32)
        constexpr int PER = C::CAP / 128;
        int mine[PER];
#pragma unroll
        for (int m2 = 0; m2 < PER; ++m2) {
          const int i = wt + 128 * m2;
          mine[m2] = i < keep ? (int)(0xFFFFFFFFu - (uint32_t)(qb[i] & 0xFFFFFFFFull)) : 0x7FFFFFFF;
        }
        wg_bar(wg);
        int* ib32 = reinterpret_cast<int*>(qb);
        const int wlo = pos - p.W + 1 > 0 ? pos - p.W + 1 : 0;
        const int wlen = pos - wlo + 1;
        int32_t* dst = p.idx + ((size_t)si.b * p.Lq + t) * p.S;
        const int ncp = pos - p.W + 1;  // candidate positions 0 .. pos - W
        const int nwords = ncp > 0 ? (ncp + 31) / 32 : 0;
        if (nwords <= 2 * C::CAP) {
          // the picks in ascending order through a bitmap of the candidate positions (in the
          // query's buffer): set their bits, then one prefix count over the words writes them;
          // the window t-W+1..t follows, all larger
          unsigned* bm = reinterpret_cast<unsigned*>(qb);
          for (int i = wt; i < nwords; i += 128) bm[i] = 0u;
          wg_bar(wg);
#pragma unroll
          for (int m2 = 0; m2 < PER; ++m2)
            if (mine[m2] != 0x7FFFFFFF) atomicOr(&bm[mine[m2] >> 5], 1u << (mine[m2] & 31));
          wg_bar(wg);
          const int per = (nwords + 127) / 128;
          const int w0 = wt * per, w1 = w0 + per < nwords ? w0 + per : nwords;
          unsigned cw = 0;
          for (int i = w0; i < w1; ++i) cw += __popc(bm[i]);
          unsigned incl = cw;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const unsigned nb = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += nb;
          }
          const int wq = (warp - 2) & 3;
          if (lane == 31) s_wsum[wg][wq] = incl;
          wg_bar(wg);
          unsigned o_pos = incl - cw;
          for (int x = 0; x < wq; ++x) o_pos += s_wsum[wg][x];
          for (int i = w0; i < w1; ++i) {
            unsigned word = bm[i];
            while (word) {
              const int bit = __ffs(word) - 1;
              word &= word - 1;
              if (o_pos < (unsigned)keep) dst[o_pos] = i * 32 + bit;
              ++o_pos;
            }
          }
          for (int i = wt; i < p.S; i += 128)
            if (i >= keep) dst[i] = i < keep + wlen ? wlo + (i - keep) : -1;
          wg_bar(wg);
          continue;
        }
        // (positions beyond the buffer's bitmap capacity) a bitonic sort of the picks
#pragma unroll
        for (int m2 = 0; m2 < 1024 / 128; ++m2) {
          const int i = wt + 128 * m2;
          ib32[i] = (i < keep && m2 < PER) ? mine[m2 < PER ? m2 : 0] : 0x7FFFFFFF;
        }
        wg_bar(wg);
        for (int k2 = 2; k2 <= 1024; k2 <<= 1) {
          for (int j2 = k2 >> 1; j2 > 0; j2 >>= 1) {
            for (int pr = wt; pr < 512; pr += 128) {
              const int i = 2 * pr - (pr & (j2 - 1));
              const int l2 = i + j2;
              const int a = ib32[i], cv = ib32[l2];
              const bool asc = (i & k2) == 0;
              if ((a > cv) == asc) { ib32[i] = cv; ib32[l2] = a; }
            }
            wg_bar(wg);
          }
        }
        const int total = keep + wlen;
        for (int i = wt; i < p.S; i += 128) dst[i] = i < keep ? ib32[i] : (i < total ? wlo + (i - keep) : -1);
        wg_bar(wg);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// =============================================================================================
// host side
// =============================================================================================
size_t workspace_bytes(int, int, int, int, int, int, int, int, size_t status_bytes) { return status_bytes; }

template <int H, int D>
static hs2_status run_t(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B, int Lq, int Lk, float c,
                        int window, int topk, hs2_bf16* out, float* lse, int32_t* idx, DevStatus* st, int sms,
                        cudaStream_t stream) {
  using FC = FaCfg<H, D>;
  using SC = ScCfg<H, D>;
  if (topk > SC::CAP - 128 || topk > 1024) return HS2_ERR_UNSUPPORTED_SHAPE;  // picks are sorted in 1024 slots
  const long long rows_total = (long long)B * Lq * H;
  if (rows_total >= (1LL << 31)) return HS2_ERR_UNSUPPORTED_SHAPE;
  CUtensorMap tmQ1, tmQ2, tmK, tmV;
  if (!make_tmap_2d(&tmQ1, Q, D, rows_total, D, 64, 128) || !make_tmap_2d(&tmQ2, Q, D, rows_total, D, 64, 256) ||
      !make_tmap_3d(&tmK, K, D, Lk, B, D, (uint64_t)Lk * D, 64, 128) ||
      !make_tmap_3d(&tmV, V, D, Lk, B, D, (uint64_t)Lk * D, 64, 128))
    return HS2_ERR_CUDA;
  PfParams p;
  p.B = B; p.Lq = Lq; p.Lk = Lk; p.H = H;
  p.off = Lk - Lq;
  p.rows_per_batch = Lq * H;
  p.items_per_batch = (Lq * H + 255) / 256;
  p.n_items = B * p.items_per_batch;
  p.c = c;
  p.W = window; p.K = topk; p.S = window + topk;
  p.out = reinterpret_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  p.idx = idx;
  p.wait_ns = wait_limit_ns();
  p.st = st;
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(fa_fwd_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, FC::SMEM);
    cudaFuncSetAttribute(score_select_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SC::SMEM);
    configured = true;
  }
  const int grid = p.n_items < sms ? p.n_items : sms;
  {
    LaunchScope ls("fa_fwd", stream);
    fa_fwd_kernel<H, D><<<grid, NT, FC::SMEM, stream>>>(tmQ1, tmK, tmV, p);
  }
  {
    LaunchScope ls("score_select", stream);
    score_select_kernel<H, D><<<grid, NT_SC, SC::SMEM, stream>>>(tmQ2, tmK, p);
  }
  return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

hs2_status run(const hs2_bf16* Q, const hs2_bf16* K, const hs2_bf16* V, int B, int Lq, int Lk, int H, int d, float c,
               int window, int topk, hs2_bf16* out, float* lse, int32_t* idx, void* ws, size_t ws_bytes, int sms,
               size_t status_bytes, cudaStream_t stream) {
  if (Lq < 1 || Lq > Lk) return HS2_ERR_UNSUPPORTED_SHAPE;
  if (ws_bytes < status_bytes) return HS2_ERR_WORKSPACE;
  DevStatus* st = reinterpret_cast<DevStatus*>(ws);
  if (H == 64 && d == 128) return run_t<64, 128>(Q, K, V, B, Lq, Lk, c, window, topk, out, lse, idx, st, sms, stream);
  if (H == 16 && d == 64) return run_t<16, 64>(Q, K, V, B, Lq, Lk, c, window, topk, out, lse, idx, st, sms, stream);
  return HS2_ERR_UNSUPPORTED_SHAPE;
}

}  // namespace prefill
}  // namespace hs2
