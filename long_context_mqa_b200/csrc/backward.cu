// Backward pass of the full layer (causal MQA attention) and of a sparse layer (attention over
// the selected tokens), for training the hybrid block: the full layers are trained natively as
// indexers (arex-research.com article "小米 MiMo 负责人罗福利公开 MiMo-V3 核心架构 HySparse2", section
// "外层 KV Bridging，内层 KV Reuse"). For a row (query, head) with key set J and output gradient dO:
//   p_j = exp2(s_j c - lse2)   (s_j = q.k_j, c = scale log2 e, lse2 the forward logsumexp / ln 2)
//   dP_j = dO.v_j, D = dO.out (= sum_j p_j dP_j), dS_j = p_j (dP_j - D)
//   dQ = scale sum_j dS_j k_j,  dK_j += scale dS_j q,  dV_j += p_j dO
// The selection is a constant of the backward pass (no gradient). K and V are shared by every head
// (MQA) and, through KV Reuse, by the full layer and its sparse layers: dK and dV are fp32 buffers
// that every layer's backward ADDS into.
//
//  prep   : D and lse2 of every row (one warp per row).
//  dq     : query-parallel. Rows of a 128-row tile are (query, head) pairs (all heads of 128 / H
//           queries, so one K/V tile serves every head). Per key tile: S = Q K^T and dP = dO V^T
//           into TMEM, dS (bf16) K-major into shared memory, dQ += dS K (the K tile read MN-major)
//           in TMEM. The next tile's S and dP are issued as soon as the softmax warps have read the
//           current ones, so they overlap the dS arithmetic. K/V through a 4-slot TMA ring.
//  dkdv   : key-parallel over (key tile, range of row tiles). Transposed tiles: S^T = K Q^T and
//           dP^T = V dO^T with the 128 keys in TMEM lanes, so a thread owns one key; P^T and dS^T
//           (bf16) are written back into TMEM over the columns just read and are the A operands of
//           dV += P^T dO and dK += dS^T Q (Q and dO tiles read MN-major). At the end of a work
//           item the CTA adds its dK, dV rows into the fp32 outputs (red.global.add.v4).
//  sparse : one CTA per query row: each tile of 128 selected K and V rows is gathered once for all
//           heads (16-byte cp.async, double-buffered); S, dP (M = 64 heads), dS and P (bf16, shared
//           memory), then dQ += dS K_sel (M = 64) and dK_sel = dS^T Q, dV_sel = P^T dO (M = 128
//           keys: the same shared-memory tiles read MN-major), scattered into dK, dV by
//           red.global.add.v4 (a key selected by many rows receives many adds).
// Warp roles of dq / dkdv (320 threads): warp 0 TMA producer, warp 1 tcgen05 issuer + TMEM owner,
// warps 2..9 the row (or key) threads: a TMEM lane (row or key) is owned by one warp of each of
// the two warpgroups, which split its 128 columns (warpgroup g takes columns 64 g .. 64 g + 63).
// Every wait is bounded and reports a timeout.
#include "decode.h"
#include "host_util.h"
#include "pair_union.cuh"
#include "tc.cuh"

namespace hs2 {
namespace bwd {

constexpr float LOG2E = 1.4426950408889634f;
constexpr int NT = 320;  // dq / dkdv: producer warp, issuer warp, two warpgroups of row (key) threads

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
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b), "f"(c), "f"(d) : "memory");
}
// untiled bulk copy global -> shared completing on `bar` (no multicast); 16-byte aligned, size % 16 == 0
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// =============================================================================================
// prep: D = <dO, out> and lse2 = lse / ln 2 per (query, head) row
// =============================================================================================
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* dO, const __nv_bfloat16* out,
                                                       const float* lse, float* Dv, float* lse2, long long n_rows) {
  griddep_wait();
  griddep_launch_dependents();
  const int lane = threadIdx.x & 31;
  const long long nw = (long long)gridDim.x * (blockDim.x / 32);
  for (long long r = blockIdx.x * (long long)(blockDim.x / 32) + threadIdx.x / 32; r < n_rows; r += nw) {
    float acc = 0.f;
    if constexpr (D == 128) {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(dO + r * D) + lane);
      const uint2 b = __ldg(reinterpret_cast<const uint2*>(out + r * D) + lane);
      const uint32_t aw[2] = {a.x, a.y}, bw[2] = {b.x, b.y};
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        acc += __uint_as_float(aw[x] << 16) * __uint_as_float(bw[x] << 16);
        acc += __uint_as_float(aw[x] & 0xFFFF0000u) * __uint_as_float(bw[x] & 0xFFFF0000u);
      }
    } else {
      const uint32_t a = __ldg(reinterpret_cast<const uint32_t*>(dO + r * D) + lane);
      const uint32_t b = __ldg(reinterpret_cast<const uint32_t*>(out + r * D) + lane);
      acc = __uint_as_float(a << 16) * __uint_as_float(b << 16) +
            __uint_as_float(a & 0xFFFF0000u) * __uint_as_float(b & 0xFFFF0000u);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      Dv[r] = acc;
      lse2[r] = lse[r] * LOG2E;
    }
  }
}

// =============================================================================================
// dq: query-parallel
// =============================================================================================
template <int D>
struct DqCfg {
  static constexpr int T_BYTES = 128 * D * 2;  // a 128-row tile of Q, dO, K or V
  static constexpr int DS_BYTES = 128 * 128 * 2;
  static constexpr int RING = 4;               // K_j, V_j, K_j+1, V_j+1
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = T_BYTES;
  static constexpr int OFF_DS = 2 * T_BYTES;
  static constexpr int OFF_RING = OFF_DS + DS_BYTES;
  static constexpr int SMEM = 1024 + OFF_RING + RING * T_BYTES;
};

// the last key tile a row tile reaches (its last query's causal row)
__device__ __forceinline__ int dq_last_tile(const BwdParams& p, int ti) {
  int q_hi = (ti * 128 + 127) / p.H;
  if (q_hi > p.Lq - 1) q_hi = p.Lq - 1;
  return (p.off + q_hi) / 128;
}

template <int H, int D>
__global__ void __launch_bounds__(NT, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                  const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BwdParams p) {
  using C = DqCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t q_full, q_empty, r_full[C::RING], r_empty[C::RING], s_full, s_empty, ds_full,
      ds_empty, dq_full, dq_empty;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const long long limit = p.wait_ns;
  constexpr uint32_t tS = 0, tP = 128, tQ = 256;
  // the D and lse2 rows come from the prep kernel before this one on the stream
  griddep_wait();
  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1); mbar_init(&q_empty, 1);
    for (int i = 0; i < C::RING; ++i) { mbar_init(&r_full[i], 1); mbar_init(&r_empty[i], 1); }
    mbar_init(&s_full, 1); mbar_init(&s_empty, 8);
    mbar_init(&ds_full, 8); mbar_init(&ds_empty, 1);
    mbar_init(&dq_full, 1); mbar_init(&dq_empty, 8);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int n_items = p.B * p.tiles_per_batch;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmdO); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
      uint32_t ri = 0;
      int it = 0;
      bool ok = true;
      for (int item = n_items - 1 - (int)blockIdx.x; item >= 0 && ok; item -= gridDim.x, ++it) {
        const int b = item / p.tiles_per_batch, ti = item % p.tiles_per_batch;
        const int r0 = b * p.rows_per_batch + ti * 128;
        const int jt = dq_last_tile(p, ti);
        if (!wait_abortable(&q_empty, (it & 1) ^ 1, limit, &abort_flag, p.st, 701)) { ok = false; break; }
        mbar_expect_tx(&q_full, 2 * C::T_BYTES);
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_2d(smem + C::OFF_Q + kb * (128 * 128), &tmQ, &q_full, kb * 64, r0);
          tma_load_2d(smem + C::OFF_DO + kb * (128 * 128), &tmdO, &q_full, kb * 64, r0);
        }
        for (int j = 0; j <= jt && ok; ++j) {
          for (int kv = 0; kv < 2; ++kv, ++ri) {
            const int s = ri % C::RING;
            if (!wait_abortable(&r_empty[s], ((ri / C::RING) & 1) ^ 1, limit, &abort_flag, p.st, 702)) { ok = false; break; }
            mbar_expect_tx(&r_full[s], C::T_BYTES);
            uint8_t* dst = smem + C::OFF_RING + s * C::T_BYTES;
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_3d(dst + kb * (128 * 128), kv == 0 ? &tmK : &tmV, &r_full[s], kb * 64, j * 128, b);
          }
        }
      }
      if (!ok)  // let the copies already issued land before the CTA exits
        for (uint32_t x = (ri > C::RING ? ri - C::RING : 0); x < ri; ++x)
          mbar_wait(&r_full[x % C::RING], (x / C::RING) & 1, limit);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ tcgen05 issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_S = idesc_bf16(128, 128, 0, 0);  // S, dP: 128 rows x 128 keys
      constexpr uint32_t IDESC_Q = idesc_bf16(128, D, 0, 1);    // dQ: dS (K-major) x K tile (MN-major)
      uint32_t ri = 0, ns = 0, nds = 0, nit = 0;
      int it = 0;
      bool ok = true;
      const uint64_t qa = sdesc(smem_u32(smem + C::OFF_Q), 16, 1024);
      const uint64_t da = sdesc(smem_u32(smem + C::OFF_DO), 16, 1024);
      const uint64_t dsa = sdesc(smem_u32(smem + C::OFF_DS), 16, 1024);
      for (int item = n_items - 1 - (int)blockIdx.x; item >= 0 && ok; item -= gridDim.x, ++it) {
        const int ti = item % p.tiles_per_batch;
        const int jt = dq_last_tile(p, ti);
        if (!wait_abortable(&q_full, it & 1, limit, &abort_flag, p.st, 710)) { ok = false; break; }
        const uint32_t base = ri;  // K_j at base + 2j, V_j at base + 2j + 1
        auto issue_sdp = [&](int j) -> bool {
          const uint32_t ks = base + 2 * j, vs = ks + 1;
          if (!wait_abortable(&r_full[ks % C::RING], (ks / C::RING) & 1, limit, &abort_flag, p.st, 711)) return false;
          if (!wait_abortable(&s_empty, (ns & 1) ^ 1, limit, &abort_flag, p.st, 712)) return false;
          tc_fence_after();
          const uint64_t ka = sdesc(smem_u32(smem + C::OFF_RING + (ks % C::RING) * C::T_BYTES), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk / 4) * (128 * 128) + (kk % 4) * 32;
            umma_ss(tmem + tS, sdesc_at(qa, o), sdesc_at(ka, o), IDESC_S, kk > 0);
          }
          if (!wait_abortable(&r_full[vs % C::RING], (vs / C::RING) & 1, limit, &abort_flag, p.st, 713)) return false;
          tc_fence_after();
          const uint64_t va = sdesc(smem_u32(smem + C::OFF_RING + (vs % C::RING) * C::T_BYTES), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk / 4) * (128 * 128) + (kk % 4) * 32;
            umma_ss(tmem + tP, sdesc_at(da, o), sdesc_at(va, o), IDESC_S, kk > 0);
          }
          umma_commit(&s_full);
          umma_commit(&r_empty[vs % C::RING]);  // V_j consumed
          ++ns;
          return true;
        };
        if (!issue_sdp(0)) { ok = false; break; }
        for (int j = 0; j <= jt; ++j) {
          // the next tile's S and dP overlap this tile's dS arithmetic
          if (j < jt && !issue_sdp(j + 1)) { ok = false; break; }
          if (!wait_abortable(&ds_full, nds & 1, limit, &abort_flag, p.st, 714)) { ok = false; break; }
          if (j == 0 && !wait_abortable(&dq_empty, (nit & 1) ^ 1, limit, &abort_flag, p.st, 715)) { ok = false; break; }
          tc_fence_after();
          const uint32_t ks = base + 2 * j;
          const uint64_t kmn = sdesc(smem_u32(smem + C::OFF_RING + (ks % C::RING) * C::T_BYTES), 128 * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk)
            umma_ss(tmem + tQ, sdesc_at(dsa, (kk / 4) * (128 * 128) + (kk % 4) * 32), sdesc_at(kmn, kk * 2048),
                    IDESC_Q, (j > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&ds_empty);
          umma_commit(&r_empty[ks % C::RING]);  // K_j consumed
          ++nds;
        }
        if (!ok) break;
        umma_commit(&dq_full);
        umma_commit(&q_empty);
        ++nit;
        ri = base + 2 * (jt + 1);
      }
    }
  } else {
    // ------------------------------------------------------------------ row threads (half a row each)
    const int quarter = warp & 3;
    const int grp = (warp - 2) >> 2;  // this warpgroup's keys: grp * 64 .. grp * 64 + 63
    const int row = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t ds_base = smem_u32(smem + C::OFF_DS);
    const float c = p.c;
    uint32_t ns = 0, nds = 0, nit = 0;
    bool ok = true;
    for (int item = n_items - 1 - (int)blockIdx.x; item >= 0 && ok; item -= gridDim.x) {
      const int b = item / p.tiles_per_batch, ti = item % p.tiles_per_batch;
      const int jt = dq_last_tile(p, ti);
      const int rloc = ti * 128 + row;
      const bool valid = rloc < p.rows_per_batch;
      const int t = p.off + (valid ? rloc / H : 0);
      const long long grow = (long long)b * p.rows_per_batch + rloc;
      const float nl2 = valid ? -__ldg(p.lse2 + grow) : 0.f;
      const float Dr = valid ? __ldg(p.Dv + grow) : 0.f;
      for (int j = 0; j <= jt; ++j) {
        if (!warp_wait(&s_full, ns & 1, limit, &abort_flag, p.st, 721)) { ok = false; break; }
        ++ns;
        tc_fence_after();
        const int kvis = valid ? t - j * 128 - grp * 64 : -1;  // keys 0..kvis of this half are in the row
        const bool masked = __any_sync(0xffffffffu, kvis < 63);
        uint32_t pk[32];  // the row's dS over this half, bf16 pairs
        {
          float sv[2][32], dv[2][32];
          tmem_ld32(tmem + lane_base + tS + grp * 64, sv[0]);
          tmem_ld32(tmem + lane_base + tS + grp * 64 + 32, sv[1]);
          tmem_ld32(tmem + lane_base + tP + grp * 64, dv[0]);
          tmem_ld32(tmem + lane_base + tP + grp * 64 + 32, dv[1]);
          tmem_ld_wait();
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2)
#pragma unroll
            for (int x = 0; x < 32; x += 2) {
              const int col = c2 * 32 + x;
              float e0, e1;
              ffma2(e0, e1, sv[c2][x], sv[c2][x + 1], c, c, nl2, nl2);
              float p0 = fast_exp2(e0), p1 = fast_exp2(e1);
              if (masked) {
                p0 = col <= kvis ? p0 : 0.f;
                p1 = col + 1 <= kvis ? p1 : 0.f;
              }
              pk[col / 2] = pack_bf16x2(p0 * (dv[c2][x] - Dr), p1 * (dv[c2][x + 1] - Dr));
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty);  // S and dP read: the next tile's may be issued
        if (!warp_wait(&ds_empty, (nds & 1) ^ 1, limit, &abort_flag, p.st, 722)) { ok = false; break; }
        // keys grp * 64.. of the row: the dS tile's K-major block grp
#pragma unroll
        for (int q = 0; q < 8; ++q)
          st_shared_v4(ds_base + grp * (128 * 128) + sw128_off(row, q), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2],
                       pk[4 * q + 3]);
        fence_async_smem();  // read by the tensor core
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_full);
        ++nds;
      }
      if (!ok) break;
      if (!warp_wait(&dq_full, nit & 1, limit, &abort_flag, p.st, 723)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c3 = 0; c3 < D / 64; ++c3) {  // this warpgroup's half of the dQ row
        const int cc = grp * (D / 64) + c3;
        float o[32];
        tmem_ld32(tmem + lane_base + tQ + cc * 32, o);
        tmem_ld_wait();
        if (valid) {
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) w[x] = pack_bf16x2(o[2 * x] * p.scale, o[2 * x + 1] * p.scale);
          uint4* dst = reinterpret_cast<uint4*>(p.dQ + grow * D + cc * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dq_empty);
      ++nit;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// =============================================================================================
// dkdv: key-parallel
// =============================================================================================
template <int D>
struct KvCfg {
  static constexpr int T_BYTES = 128 * D * 2;
  static constexpr int RING = 4;  // Q_i, dO_i, Q_i+1, dO_i+1
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = T_BYTES;
  static constexpr int OFF_RING = 2 * T_BYTES;
  static constexpr int SMEM = 1024 + OFF_RING + RING * T_BYTES;
};

// the row tiles [rt0, rt1) of work item `item` (sequence b, key tile kt, chunk of row tiles);
// rows of queries before the key tile's first key never reach it
struct KvItem {
  int b, kt, rt0, rt1;
};
__device__ __forceinline__ KvItem kv_item(const BwdParams& p, int item) {
  KvItem w;
  const int per_b = p.kv_tiles * p.n_chunks;
  w.b = item / per_b;
  const int rem = item % per_b;
  w.kt = rem / p.n_chunks;
  const int ch = rem % p.n_chunks;
  const int q0 = w.kt * 128 - p.off;  // first query position reaching the tile's first key
  const int rt_min = q0 > 0 ? (int)(((long long)q0 * p.H) / 128) : 0;
  w.rt0 = ch * p.chunk > rt_min ? ch * p.chunk : rt_min;
  w.rt1 = (ch + 1) * p.chunk < p.tiles_per_batch ? (ch + 1) * p.chunk : p.tiles_per_batch;
  return w;
}

template <int H, int D>
__global__ void __launch_bounds__(NT, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
                    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, BwdParams p) {
  using C = KvCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t kv_in_full, kv_in_empty, r_full[C::RING], r_empty[C::RING], s_full, ps_full,
      step_done, kv_full, kv_empty;
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  // lse2 and D of the 128 rows of the Q tile in ring slot s (loaded with it)
  __shared__ __align__(16) float s_side[C::RING][2][128];
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const long long limit = p.wait_ns;
  // TMEM: S^T (P^T packed into its first 64 columns once read), dP^T (dS^T likewise), dV, dK
  constexpr uint32_t tS = 0, tP = 128, tV = 256, tK = 256 + D;
  griddep_wait();
  if (threadIdx.x == 0) {
    mbar_init(&kv_in_full, 1); mbar_init(&kv_in_empty, 1);
    for (int i = 0; i < C::RING; ++i) { mbar_init(&r_full[i], 1); mbar_init(&r_empty[i], 1); }
    mbar_init(&s_full, 1); mbar_init(&ps_full, 8); mbar_init(&step_done, 1);
    mbar_init(&kv_full, 1); mbar_init(&kv_empty, 8);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const int n_items = p.B * p.kv_tiles * p.n_chunks;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmQ); tma_prefetch_desc(&tmdO); tma_prefetch_desc(&tmK); tma_prefetch_desc(&tmV);
      uint32_t ri = 0;
      int it = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const KvItem w = kv_item(p, item);
        if (w.rt0 >= w.rt1) continue;
        if (!wait_abortable(&kv_in_empty, (it & 1) ^ 1, limit, &abort_flag, p.st, 731)) { ok = false; break; }
        mbar_expect_tx(&kv_in_full, 2 * C::T_BYTES);
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_3d(smem + C::OFF_K + kb * (128 * 128), &tmK, &kv_in_full, kb * 64, w.kt * 128, w.b);
          tma_load_3d(smem + C::OFF_V + kb * (128 * 128), &tmV, &kv_in_full, kb * 64, w.kt * 128, w.b);
        }
        ++it;
        for (int rt = w.rt0; rt < w.rt1 && ok; ++rt) {
          const int r0 = w.b * p.rows_per_batch + rt * 128;
          for (int which = 0; which < 2; ++which, ++ri) {
            const int s = ri % C::RING;
            if (!wait_abortable(&r_empty[s], ((ri / C::RING) & 1) ^ 1, limit, &abort_flag, p.st, 732)) { ok = false; break; }
            // with the Q tile: the rows' lse2 and D (the arrays are padded by a tile at the end)
            mbar_expect_tx(&r_full[s], C::T_BYTES + (which == 0 ? 1024u : 0u));
            uint8_t* dst = smem + C::OFF_RING + s * C::T_BYTES;
            for (int kb = 0; kb < D / 64; ++kb)
              tma_load_2d(dst + kb * (128 * 128), which == 0 ? &tmQ : &tmdO, &r_full[s], kb * 64, r0);
            if (which == 0) {
              bulk_load(&s_side[s][0][0], p.lse2 + r0, 512, &r_full[s]);
              bulk_load(&s_side[s][1][0], p.Dv + r0, 512, &r_full[s]);
            }
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
      constexpr uint32_t IDESC_T = idesc_bf16(128, 128, 0, 0);  // S^T, dP^T: 128 keys x 128 rows
      constexpr uint32_t IDESC_KV = idesc_bf16(128, D, 0, 1);   // dV, dK: A in TMEM, B MN-major
      uint32_t ri = 0, nstep = 0, nps = 0, nit = 0;
      int it = 0;
      bool ok = true;
      const uint64_t ka = sdesc(smem_u32(smem + C::OFF_K), 16, 1024);
      const uint64_t va = sdesc(smem_u32(smem + C::OFF_V), 16, 1024);
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const KvItem w = kv_item(p, item);
        if (w.rt0 >= w.rt1) continue;
        if (!wait_abortable(&kv_in_full, it & 1, limit, &abort_flag, p.st, 740)) { ok = false; break; }
        ++it;
        const uint32_t base = ri;
        const int n = w.rt1 - w.rt0;
        for (int i = 0; i < n; ++i) {
          const uint32_t qs = base + 2 * i, ds = qs + 1;
          if (!wait_abortable(&r_full[qs % C::RING], (qs / C::RING) & 1, limit, &abort_flag, p.st, 741)) { ok = false; break; }
          // the previous step's dV, dK read P^T, dS^T from the columns S^T, dP^T overwrite
          if (nstep > 0 && !wait_abortable(&step_done, (nstep - 1) & 1, limit, &abort_flag, p.st, 742)) { ok = false; break; }
          tc_fence_after();
          const uint32_t qaddr = smem_u32(smem + C::OFF_RING + (qs % C::RING) * C::T_BYTES);
          const uint32_t daddr = smem_u32(smem + C::OFF_RING + (ds % C::RING) * C::T_BYTES);
          const uint64_t qk = sdesc(qaddr, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk / 4) * (128 * 128) + (kk % 4) * 32;
            umma_ss(tmem + tS, sdesc_at(ka, o), sdesc_at(qk, o), IDESC_T, kk > 0);
          }
          if (!wait_abortable(&r_full[ds % C::RING], (ds / C::RING) & 1, limit, &abort_flag, p.st, 743)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dk = sdesc(daddr, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t o = (kk / 4) * (128 * 128) + (kk % 4) * 32;
            umma_ss(tmem + tP, sdesc_at(va, o), sdesc_at(dk, o), IDESC_T, kk > 0);
          }
          umma_commit(&s_full);
          if (!wait_abortable(&ps_full, nps & 1, limit, &abort_flag, p.st, 744)) { ok = false; break; }
          ++nps;
          if (i == 0 && !wait_abortable(&kv_empty, (nit & 1) ^ 1, limit, &abort_flag, p.st, 745)) { ok = false; break; }
          tc_fence_after();
          const uint64_t dmn = sdesc(daddr, 128 * 128, 1024), qmn = sdesc(qaddr, 128 * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            // rows 64 g .. 64 g + 63 of the tile (K steps 4 g .. 4 g + 3) were packed by warpgroup g
            // into columns 64 g .. 64 g + 31 of the S^T / dP^T regions
            const uint32_t acol = (kk / 4) * 64 + (kk % 4) * 8;
            umma_ts(tmem + tV, tmem + tS + acol, sdesc_at(dmn, kk * 2048), IDESC_KV, (i > 0 || kk > 0) ? 1u : 0u);
            umma_ts(tmem + tK, tmem + tP + acol, sdesc_at(qmn, kk * 2048), IDESC_KV, (i > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&r_empty[qs % C::RING]);
          umma_commit(&r_empty[ds % C::RING]);
          umma_commit(&step_done);
          ++nstep;
        }
        if (!ok) break;
        umma_commit(&kv_full);
        umma_commit(&kv_in_empty);
        ++nit;
        ri = base + 2 * n;
      }
    }
  } else {
    // ------------------------------------------------------------------ key threads (half a key's columns each)
    const int quarter = warp & 3;
    const int grp = (warp - 2) >> 2;  // this warpgroup's columns (rows of the tile): grp * 64 ..
    const int krow = quarter * 32 + lane;
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float c = p.c;
    uint32_t ns = 0, nit = 0, ri = 0;
    bool ok = true;
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const KvItem w = kv_item(p, item);
      if (w.rt0 >= w.rt1) continue;
      const int kglob = w.kt * 128 + krow;
      for (int rt = w.rt0; rt < w.rt1; ++rt, ri += 2) {
        if (!warp_wait(&s_full, ns & 1, limit, &abort_flag, p.st, 751)) { ok = false; break; }
        ++ns;
        tc_fence_after();
        // the tile's columns: rows rt * 128 + col, their lse2 and D staged with the Q tile (the
        // S^T MMA waited for that slot), their query positions; a row past the sequence sees no key
        if (!warp_wait(&r_full[ri % C::RING], (ri / C::RING) & 1, limit, &abort_flag, p.st, 753)) { ok = false; break; }
        const float* l2c = &s_side[ri % C::RING][0][0];
        const float* dcol = &s_side[ri % C::RING][1][0];
        const int rbase = rt * 128;
        auto t_of = [&](int col) { return rbase + col < p.rows_per_batch ? p.off + (rbase + col) / H : -1; };
        // 32 columns at a time: their P^T and dS^T packed two per column into the first half of
        // this warpgroup's 64-column window (chunk c2 -> columns 16 c2 .., all already read)
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          float sv[32], dv[32];
          tmem_ld32(tmem + lane_base + tS + grp * 64 + c2 * 32, sv);
          tmem_ld32(tmem + lane_base + tP + grp * 64 + c2 * 32, dv);
          tmem_ld_wait();
          float pp[16], dd[16];  // bf16 pairs, as 32-bit patterns
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const int col = grp * 64 + c2 * 32 + x;
            float e0, e1;
            ffma2(e0, e1, sv[x], sv[x + 1], c, c, -l2c[col], -l2c[col + 1]);
            const float p0 = kglob <= t_of(col) ? fast_exp2(e0) : 0.f;
            const float p1 = kglob <= t_of(col + 1) ? fast_exp2(e1) : 0.f;
            pp[x / 2] = __uint_as_float(pack_bf16x2(p0, p1));
            dd[x / 2] = __uint_as_float(pack_bf16x2(p0 * (dv[x] - dcol[col]), p1 * (dv[x + 1] - dcol[col + 1])));
          }
          tmem_st16(tmem + lane_base + tS + grp * 64 + c2 * 16, pp);
          tmem_st16(tmem + lane_base + tP + grp * 64 + c2 * 16, dd);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ps_full);
      }
      if (!ok) break;
      if (!warp_wait(&kv_full, nit & 1, limit, &abort_flag, p.st, 752)) { ok = false; break; }
      tc_fence_after();
      const bool kv = kglob < p.Lk;
      float* dKr = p.dK + ((long long)w.b * p.Lk + kglob) * D;
      float* dVr = p.dV + ((long long)w.b * p.Lk + kglob) * D;
#pragma unroll
      for (int c3 = 0; c3 < D / 64; ++c3) {  // this warpgroup's half of the key's dK, dV rows
        const int cc = grp * (D / 64) + c3;
        float a[32], v[32];
        tmem_ld32(tmem + lane_base + tK + cc * 32, a);
        tmem_ld32(tmem + lane_base + tV + cc * 32, v);
        tmem_ld_wait();
        if (kv) {
#pragma unroll
          for (int x = 0; x < 32; x += 4) {
            red_add_v4(dKr + cc * 32 + x, a[x] * p.scale, a[x + 1] * p.scale, a[x + 2] * p.scale, a[x + 3] * p.scale);
            red_add_v4(dVr + cc * 32 + x, v[x], v[x + 1], v[x + 2], v[x + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&kv_empty);
      ++nit;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// =============================================================================================
// sparse layer backward: one CTA per query row, 128 threads
// =============================================================================================
constexpr int MH = 64;  // MMA rows of the head side (heads zero-padded to 64)

template <int D>
struct SbCfg {
  static constexpr int Q_BYTES = MH * D * 2;    // Q, dO: K-major [64 x D]
  static constexpr int P_BYTES = MH * 128 * 2;  // P, dS: K-major [64 heads x 128 keys]
  static constexpr int KT_BYTES = 128 * D * 2;  // a gathered K (or V) tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = Q_BYTES;
  static constexpr int OFF_P = 2 * Q_BYTES;
  static constexpr int OFF_DS = OFF_P + P_BYTES;
  static constexpr int OFF_KV = ((OFF_DS + P_BYTES + 1023) / 1024) * 1024;  // 2 stages x (K, V)
  static constexpr int SMEM = 1024 + OFF_KV + 4 * KT_BYTES;
};

template <int H, int D>
__global__ void __launch_bounds__(128, 1) sparse_bwd_kernel(BwdParams p) {
  using C = SbCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ unsigned vmask[2][4];
  __shared__ float s_nl2[MH], s_D[MH];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // TMEM: S (M = 64), later dV_sel (M = 128); dP (M = 64); dQ (M = 64); dK_sel (M = 128)
  constexpr uint32_t tS = 0, tP = 128, tQ = 256, tK = 384;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  const int prow = warp * 16 + (lane & 15);  // head row this lane's pair works on
  const bool upper = lane >= 16;
  griddep_wait();
  griddep_launch_dependents();
  if (tid == 0) { mbar_init(&mma_bar, 1); fence_mbar_init(); }
  if (warp == 0) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const float c = p.c;
  const int ntiles = (p.S + 127) / 128;
  const int n_rows = p.B * p.Lq;
  uint32_t phase = 0;
  bool ok = true, bad = false;
  auto mma_wait = [&](unsigned where) -> bool {
    bool w_ok = true;
    if (tid == 0) w_ok = mbar_wait(&mma_bar, phase, p.wait_ns);
    phase ^= 1;
    if (!__syncthreads_and(w_ok)) {
      if (tid == 0) report_status(p.st, kStatusTimeout, where);
      return false;
    }
    tc_fence_after();
    return true;
  };
  for (int r = blockIdx.x; r < n_rows && ok; r += gridDim.x) {
    const int b = r / p.Lq;
    const int32_t* idx_row = p.idx + (size_t)r * p.S;
    const __nv_bfloat16* Kb = p.K + (size_t)b * p.Lk * D;
    const __nv_bfloat16* Vb = p.V + (size_t)b * p.Lk * D;
    // ---- Q and dO rows -> shared (K-major, 128B swizzle), padding rows zero; per-head D, -lse2
    for (int cidx = tid; cidx < MH * D / 8; cidx += 128) {
      const int row = cidx / (D / 8), ch = cidx % (D / 8);
      const uint32_t off = (ch / 8) * (MH * 128) + sw128_off(row, ch % 8);
      if (row < H) {
        cp_async_16(smem_u32(smem + C::OFF_Q) + off, p.Q + ((size_t)r * H + row) * D + ch * 8, true);
        cp_async_16(smem_u32(smem + C::OFF_DO) + off, p.dO + ((size_t)r * H + row) * D + ch * 8, true);
      } else {
        st_shared_v4(smem_u32(smem + C::OFF_Q) + off, 0u, 0u, 0u, 0u);
        st_shared_v4(smem_u32(smem + C::OFF_DO) + off, 0u, 0u, 0u, 0u);
      }
    }
    if (tid < MH) {
      s_nl2[tid] = tid < H ? -__ldg(p.lse2 + (size_t)r * H + tid) : 0.f;
      s_D[tid] = tid < H ? __ldg(p.Dv + (size_t)r * H + tid) : 0.f;
    }
    // gathers the selected K and V rows of tile t into stage t & 1 (16 lanes per 256-byte row,
    // the row's index passed by shuffle from the lane that read it); returns this thread's key
    auto gather = [&](int t) -> int {
      constexpr int LPR = D * 2 / 16, RPS = 32 / LPR;
      const int slot = t * 128 + tid;
      int j = slot < p.S ? idx_row[slot] : -1;
      const bool valid = j >= 0 && j < p.Lk;
      if (j != -1 && !valid) bad = true;
      if (!valid) j = -1;
      const unsigned m = __ballot_sync(0xffffffffu, valid);
      if (lane == 0) vmask[t & 1][warp] = m;
      const uint32_t kd = smem_u32(smem + C::OFF_KV + (t & 1) * 2 * C::KT_BYTES), vd = kd + C::KT_BYTES;
      const int sub = lane / LPR, ch = lane % LPR;
#pragma unroll
      for (int it = 0; it < 32 / RPS; ++it) {
        const int rr = it * RPS + sub;
        const int kr = __shfl_sync(0xffffffffu, j, rr);
        const uint32_t off = (ch / 8) * (128 * 128) + sw128_off(warp * 32 + rr, ch % 8);
        const size_t src = (size_t)(kr >= 0 ? kr : 0) * D + ch * 8;
        cp_async_16(kd + off, Kb + src, kr >= 0);
        cp_async_16(vd + off, Vb + src, kr >= 0);
      }
      cp_async_commit();
      return j;
    };
    int j_cur = gather(0);
    for (int t = 0; t < ntiles && ok; ++t) {
      int j_next = -1;
      if (t + 1 < ntiles) {
        j_next = gather(t + 1);  // the other stage was last read by tile t - 1's MMAs (complete)
        asm volatile("cp.async.wait_group 1;" ::: "memory");
      } else {
        cp_async_wait_all();
      }
      fence_async_smem();
      __syncthreads();
      const uint32_t kst = smem_u32(smem + C::OFF_KV + (t & 1) * 2 * C::KT_BYTES), vst = kst + C::KT_BYTES;
      // ---- S = Q K_sel^T, dP = dO V_sel^T (M = 64 heads, N = 128 keys)
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t IDESC = idesc_bf16(MH, 128, 0, 0);
        const uint64_t qa = sdesc(smem_u32(smem + C::OFF_Q), 16, 1024), da = sdesc(smem_u32(smem + C::OFF_DO), 16, 1024);
        const uint64_t ka = sdesc(kst, 16, 1024), va = sdesc(vst, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t oa = (kk / 4) * (MH * 128) + (kk % 4) * 32, ob = (kk / 4) * (128 * 128) + (kk % 4) * 32;
          umma_ss(tmem + tS, sdesc_at(qa, oa), sdesc_at(ka, ob), IDESC, kk > 0);
          umma_ss(tmem + tP, sdesc_at(da, oa), sdesc_at(va, ob), IDESC, kk > 0);
        }
        umma_commit(&mma_bar);
      }
      if (!mma_wait(801)) { ok = false; break; }
      // ---- P and dS rows (bf16, K-major [64 heads x 128 keys]); lane l < 16 keeps keys 0..63
      // of head row prow, lane l + 16 takes keys 64..127 of the same row
      {
        const float nl2 = s_nl2[prow], Dr = s_D[prow];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          // columns h2 * 32.. (kept by lanes < 16) and 64 + h2 * 32.. (taken by lanes >= 16)
          float s_lo[32], s_hi[32], d_lo[32], d_hi[32];
          tmem_ld32(tmem + lane_base + tS + h2 * 32, s_lo);
          tmem_ld32(tmem + lane_base + tS + 64 + h2 * 32, s_hi);
          tmem_ld32(tmem + lane_base + tP + h2 * 32, d_lo);
          tmem_ld32(tmem + lane_base + tP + 64 + h2 * 32, d_hi);
          tmem_ld_wait();
          float sv[32], dv[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const float hs = __shfl_xor_sync(0xffffffffu, s_hi[x], 16);
            const float hd = __shfl_xor_sync(0xffffffffu, d_hi[x], 16);
            sv[x] = upper ? hs : s_lo[x];
            dv[x] = upper ? hd : d_lo[x];
          }
          const unsigned mk = vmask[t & 1][(upper ? 2 : 0) + h2];
          uint32_t pp[16], dd[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float e0, e1;
            ffma2(e0, e1, sv[x], sv[x + 1], c, c, nl2, nl2);
            const float p0 = (mk >> x) & 1u && prow < H ? fast_exp2(e0) : 0.f;
            const float p1 = (mk >> (x + 1)) & 1u && prow < H ? fast_exp2(e1) : 0.f;
            pp[x / 2] = pack_bf16x2(p0, p1);
            dd[x / 2] = pack_bf16x2(p0 * (dv[x] - Dr), p1 * (dv[x + 1] - Dr));
          }
          const uint32_t pb = smem_u32(smem + C::OFF_P) + (upper ? MH * 128 : 0);
          const uint32_t db = smem_u32(smem + C::OFF_DS) + (upper ? MH * 128 : 0);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            st_shared_v4(pb + sw128_off(prow, h2 * 4 + q), pp[4 * q], pp[4 * q + 1], pp[4 * q + 2], pp[4 * q + 3]);
            st_shared_v4(db + sw128_off(prow, h2 * 4 + q), dd[4 * q], dd[4 * q + 1], dd[4 * q + 2], dd[4 * q + 3]);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      // ---- dQ += dS K_sel (M = 64, N = D); dK_sel = dS^T Q, dV_sel = P^T dO (M = 128 keys, N = D)
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t IDESC_Q = idesc_bf16(MH, D, 0, 1);
        constexpr uint32_t IDESC_KV = idesc_bf16(128, D, 1, 1);
        const uint64_t dsk = sdesc(smem_u32(smem + C::OFF_DS), 16, 1024);
        const uint64_t kmn = sdesc(kst, 128 * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          umma_ss(tmem + tQ, sdesc_at(dsk, (kk / 4) * (MH * 128) + (kk % 4) * 32), sdesc_at(kmn, kk * 2048), IDESC_Q,
                  (t > 0 || kk > 0) ? 1u : 0u);
        const uint64_t dsm = sdesc(smem_u32(smem + C::OFF_DS), MH * 128, 1024);
        const uint64_t pm = sdesc(smem_u32(smem + C::OFF_P), MH * 128, 1024);
        const uint64_t qm = sdesc(smem_u32(smem + C::OFF_Q), MH * 128, 1024);
        const uint64_t dom = sdesc(smem_u32(smem + C::OFF_DO), MH * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < MH / 16; ++kk) {
          umma_ss(tmem + tK, sdesc_at(dsm, kk * 2048), sdesc_at(qm, kk * 2048), IDESC_KV, kk > 0);
          umma_ss(tmem + tS, sdesc_at(pm, kk * 2048), sdesc_at(dom, kk * 2048), IDESC_KV, kk > 0);
        }
        umma_commit(&mma_bar);
      }
      if (!mma_wait(802)) { ok = false; break; }
      // ---- scatter: thread tid owns key row tid of the tile (its gathered index j_cur). The TMEM
      // loads are warp-collective (.sync.aligned): every lane executes them, whatever its slot
      {
        float* dKr = p.dK + ((size_t)b * p.Lk + (j_cur >= 0 ? j_cur : 0)) * D;
        float* dVr = p.dV + ((size_t)b * p.Lk + (j_cur >= 0 ? j_cur : 0)) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          float a[32], v[32];
          tmem_ld32(tmem + lane_base + tK + cc * 32, a);
          tmem_ld32(tmem + lane_base + tS + cc * 32, v);
          tmem_ld_wait();
          if (j_cur >= 0) {
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
              red_add_v4(dKr + cc * 32 + x, a[x] * p.scale, a[x + 1] * p.scale, a[x + 2] * p.scale, a[x + 3] * p.scale);
              red_add_v4(dVr + cc * 32 + x, v[x], v[x + 1], v[x + 2], v[x + 3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncthreads();  // TMEM S / dK_sel and the shared tiles are reused by the next tile
      j_cur = j_next;
    }
    cp_async_wait_all();
    if (!ok) break;
    // ---- dQ rows: lane l < 16 of warp q owns head row 16 q + l
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      float o[32];
      tmem_ld32(tmem + lane_base + tQ + cc * 32, o);
      tmem_ld_wait();
      const int head = warp * 16 + lane;
      if (lane < 16 && head < H) {
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) w[x] = pack_bf16x2(o[2 * x] * p.scale, o[2 * x + 1] * p.scale);
        uint4* dst = reinterpret_cast<uint4*>(p.dQ + ((size_t)r * H + head) * D + cc * 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();  // the next row's first dQ MMA overwrites the accumulator
  }
  cp_async_wait_all();
  if (__syncthreads_or(bad) && tid == 0) report_status(p.st, kStatusBounds, 803);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// =============================================================================================
// sparse layer backward, two adjacent query rows per CTA (64 heads): over the union of their
// selections, with M = 128 MMAs (both rows' heads) and one add per key for both rows
// =============================================================================================
template <int D>
struct PairCfg {
  static constexpr int T_BYTES = 128 * D * 2;   // Q / dO of the two rows, or a gathered K / V tile
  static constexpr int P_BYTES = 128 * 128 * 2;  // P, dS: K-major [128 rows x 128 keys]
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_DO = T_BYTES;
  static constexpr int OFF_P = 2 * T_BYTES;
  static constexpr int OFF_DS = OFF_P + P_BYTES;
  static constexpr int OFF_K = OFF_DS + P_BYTES;
  static constexpr int OFF_V = OFF_K + T_BYTES;
  static constexpr int OFF_UKEY = OFF_V + T_BYTES;           // int32 [PAIR_MAX]
  static constexpr int OFF_UFLAG = OFF_UKEY + PAIR_MAX * 4;  // uint8 [PAIR_MAX]
  static constexpr int SMEM = 1024 + OFF_UFLAG + PAIR_MAX;
};

template <int D>
__global__ void __launch_bounds__(128, 1) sparse_bwd_pair_kernel(BwdParams p) {
  using C = PairCfg<D>;
  constexpr int H = 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  int32_t* ukey = reinterpret_cast<int32_t*>(smem + C::OFF_UKEY);
  uint8_t* uflag = smem + C::OFF_UFLAG;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ float s_nl2[128], s_D[128];
  __shared__ int s_warp[4], s_n[8];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // TMEM: S (later dV_sel), dP, dQ of the two rows, dK_sel
  constexpr uint32_t tS = 0, tP = 128, tQ = 256, tK = 384;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
  griddep_wait();
  griddep_launch_dependents();
  if (tid == 0) { mbar_init(&mma_bar, 1); fence_mbar_init(); }
  if (warp == 0) { tmem_alloc(&tmem_base, 512); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const float c = p.c;
  const int pairs_per_b = (p.Lq + 1) / 2;
  const int n_pairs = p.B * pairs_per_b;
  uint32_t phase = 0;
  bool ok = true, bad = false;
  auto mma_wait = [&](unsigned where) -> bool {
    bool w_ok = true;
    if (tid == 0) w_ok = mbar_wait(&mma_bar, phase, p.wait_ns);
    phase ^= 1;
    if (!__syncthreads_and(w_ok)) {
      if (tid == 0) report_status(p.st, kStatusTimeout, where);
      return false;
    }
    tc_fence_after();
    return true;
  };
  for (int pr = blockIdx.x; pr < n_pairs && ok; pr += gridDim.x) {
    const int b = pr / pairs_per_b;
    const int i0 = 2 * (pr % pairs_per_b);
    const bool two = i0 + 1 < p.Lq;
    const int r0 = b * p.Lq + i0, r1 = r0 + 1;
    const __nv_bfloat16* Kb = p.K + (size_t)b * p.Lk * D;
    const __nv_bfloat16* Vb = p.V + (size_t)b * p.Lk * D;
    // ---- Q and dO of both rows -> shared (K-major, 128B swizzle): row m = 64 * (row of the pair) + head
    for (int cidx = tid; cidx < 128 * D / 8; cidx += 128) {
      const int m = cidx / (D / 8), ch = cidx % (D / 8);
      const uint32_t off = (ch / 8) * (128 * 128) + sw128_off(m, ch % 8);
      const bool have = m < H || two;
      const size_t src = ((size_t)(m < H ? r0 : r1) * H + (m & (H - 1))) * D + ch * 8;
      if (have) {
        cp_async_16(smem_u32(smem + C::OFF_Q) + off, p.Q + src, true);
        cp_async_16(smem_u32(smem + C::OFF_DO) + off, p.dO + src, true);
      } else {
        st_shared_v4(smem_u32(smem + C::OFF_Q) + off, 0u, 0u, 0u, 0u);
        st_shared_v4(smem_u32(smem + C::OFF_DO) + off, 0u, 0u, 0u, 0u);
      }
    }
    cp_async_commit();
    {
      const int m = tid;  // 128 rows, one per thread
      const bool have = m < H || two;
      const size_t g = (size_t)(m < H ? r0 : r1) * H + (m & (H - 1));
      s_nl2[m] = have ? -__ldg(p.lse2 + g) : 0.f;
      s_D[m] = have ? __ldg(p.Dv + g) : 0.f;
    }
    // ---- the union of the two rows' selections. Lists that are strictly ascending with any -1
    // slots at the tail (the full layer's output) are merged without duplicates (a key in both
    // rows gets both bits); any other lists are concatenated (each slot once, as the forward
    // counts them). Out-of-range keys are reported and left out.
    // the two index lists, staged in the P buffer (free until the first tile's softmax), and their
    // union into ukey / uflag
    const int U = pair_union(p.idx, p.S, p.Lk, r0, two, reinterpret_cast<int32_t*>(smem + C::OFF_P), ukey, uflag,
                             s_warp, s_n, bad);
    const int ntiles = (U + 127) / 128;
    cp_async_wait_all();
    __syncthreads();
    for (int t = 0; t < ntiles && ok; ++t) {
      // ---- gather the tile's K and V rows (16 lanes per 256-byte row, the key by shuffle)
      const int slot = t * 128 + tid;
      const int j = slot < U ? ukey[slot] : -1;
      const unsigned fl = slot < U ? uflag[slot] : 0u;
      {
        constexpr int LPR = D * 2 / 16, RPS = 32 / LPR;
        const int sub = lane / LPR, ch = lane % LPR;
        const uint32_t kd = smem_u32(smem + C::OFF_K), vd = smem_u32(smem + C::OFF_V);
#pragma unroll
        for (int it = 0; it < 32 / RPS; ++it) {
          const int rr = it * RPS + sub;
          const int kr = __shfl_sync(0xffffffffu, j, rr);
          const uint32_t off = (ch / 8) * (128 * 128) + sw128_off(warp * 32 + rr, ch % 8);
          const size_t src = (size_t)(kr >= 0 ? kr : 0) * D + ch * 8;
          cp_async_16(kd + off, Kb + src, kr >= 0);
          cp_async_16(vd + off, Vb + src, kr >= 0);
        }
        cp_async_commit();
      }
      // the tile's membership bits per key, for every row thread: keys 32 q .. of row q's warp
      __shared__ unsigned s_m0[4], s_m1[4];
      {
        const unsigned b0 = __ballot_sync(0xffffffffu, (fl & 1u) != 0), b1 = __ballot_sync(0xffffffffu, (fl & 2u) != 0);
        if (lane == 0) { s_m0[warp] = b0; s_m1[warp] = b1; }
      }
      cp_async_wait_all();
      fence_async_smem();
      __syncthreads();
      // ---- S = Q K_sel^T, dP = dO V_sel^T (M = 128 rows: both rows' heads, N = 128 keys)
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t IDESC = idesc_bf16(128, 128, 0, 0);
        const uint64_t qa = sdesc(smem_u32(smem + C::OFF_Q), 16, 1024), da = sdesc(smem_u32(smem + C::OFF_DO), 16, 1024);
        const uint64_t ka = sdesc(smem_u32(smem + C::OFF_K), 16, 1024), va = sdesc(smem_u32(smem + C::OFF_V), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t o = (kk / 4) * (128 * 128) + (kk % 4) * 32;
          umma_ss(tmem + tS, sdesc_at(qa, o), sdesc_at(ka, o), IDESC, kk > 0);
          umma_ss(tmem + tP, sdesc_at(da, o), sdesc_at(va, o), IDESC, kk > 0);
        }
        umma_commit(&mma_bar);
      }
      if (!mma_wait(811)) { ok = false; break; }
      // ---- P and dS rows (bf16, K-major [128 rows x 128 keys]); thread tid owns row tid
      {
        const int m = tid;
        const bool row1 = m >= H;
        const float nl2 = s_nl2[m], Dr = s_D[m];
        const uint32_t pb = smem_u32(smem + C::OFF_P), db = smem_u32(smem + C::OFF_DS);
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {  // keys 32 cc .. 32 cc + 31
          float sv[32], dv[32];
          tmem_ld32(tmem + lane_base + tS + cc * 32, sv);
          tmem_ld32(tmem + lane_base + tP + cc * 32, dv);
          tmem_ld_wait();
          const unsigned mk = (row1 ? s_m1[cc] : s_m0[cc]);
          uint32_t pp[16], dd[16];
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            float e0, e1;
            ffma2(e0, e1, sv[x], sv[x + 1], c, c, nl2, nl2);
            const float p0 = (mk >> x) & 1u ? fast_exp2(e0) : 0.f;
            const float p1 = (mk >> (x + 1)) & 1u ? fast_exp2(e1) : 0.f;
            pp[x / 2] = pack_bf16x2(p0, p1);
            dd[x / 2] = pack_bf16x2(p0 * (dv[x] - Dr), p1 * (dv[x + 1] - Dr));
          }
          // keys 32 cc .. in block cc / 2 (64 keys = one 128-byte row), chunks 4 (cc % 2) ..
          const uint32_t o = (cc / 2) * (128 * 128);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            st_shared_v4(pb + o + sw128_off(m, (cc % 2) * 4 + q), pp[4 * q], pp[4 * q + 1], pp[4 * q + 2], pp[4 * q + 3]);
            st_shared_v4(db + o + sw128_off(m, (cc % 2) * 4 + q), dd[4 * q], dd[4 * q + 1], dd[4 * q + 2], dd[4 * q + 3]);
          }
        }
      }
      fence_async_smem();
      tc_fence_before();
      __syncthreads();
      // ---- dQ += dS K_sel; dK_sel = dS^T Q, dV_sel = P^T dO (M = 128 keys, K = 128 rows)
      if (tid == 0) {
        tc_fence_after();
        constexpr uint32_t IDESC_Q = idesc_bf16(128, D, 0, 1);
        constexpr uint32_t IDESC_KV = idesc_bf16(128, D, 1, 1);
        const uint64_t dsk = sdesc(smem_u32(smem + C::OFF_DS), 16, 1024);
        const uint64_t kmn = sdesc(smem_u32(smem + C::OFF_K), 128 * 128, 1024);
        const uint64_t dsm = sdesc(smem_u32(smem + C::OFF_DS), 128 * 128, 1024);
        const uint64_t pm = sdesc(smem_u32(smem + C::OFF_P), 128 * 128, 1024);
        const uint64_t qm = sdesc(smem_u32(smem + C::OFF_Q), 128 * 128, 1024);
        const uint64_t dom = sdesc(smem_u32(smem + C::OFF_DO), 128 * 128, 1024);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          umma_ss(tmem + tQ, sdesc_at(dsk, (kk / 4) * (128 * 128) + (kk % 4) * 32), sdesc_at(kmn, kk * 2048), IDESC_Q,
                  (t > 0 || kk > 0) ? 1u : 0u);
          umma_ss(tmem + tK, sdesc_at(dsm, kk * 2048), sdesc_at(qm, kk * 2048), IDESC_KV, kk > 0);
          umma_ss(tmem + tS, sdesc_at(pm, kk * 2048), sdesc_at(dom, kk * 2048), IDESC_KV, kk > 0);
        }
        umma_commit(&mma_bar);
      }
      if (!mma_wait(812)) { ok = false; break; }
      // ---- scatter: thread tid owns key row tid of the tile; every lane runs the TMEM loads
      {
        float* dKr = p.dK + ((size_t)b * p.Lk + (j >= 0 ? j : 0)) * D;
        float* dVr = p.dV + ((size_t)b * p.Lk + (j >= 0 ? j : 0)) * D;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          float a[32], v[32];
          tmem_ld32(tmem + lane_base + tK + cc * 32, a);
          tmem_ld32(tmem + lane_base + tS + cc * 32, v);
          tmem_ld_wait();
          if (j >= 0) {
#pragma unroll
            for (int x = 0; x < 32; x += 4) {
              red_add_v4(dKr + cc * 32 + x, a[x] * p.scale, a[x + 1] * p.scale, a[x + 2] * p.scale, a[x + 3] * p.scale);
              red_add_v4(dVr + cc * 32 + x, v[x], v[x + 1], v[x + 2], v[x + 3]);
            }
          }
        }
      }
      tc_fence_before();
      __syncthreads();  // TMEM S / dK_sel and the shared tiles are reused by the next tile
    }
    if (!ok) break;
    // ---- dQ rows: thread tid owns row tid (row tid / 64 of the pair, head tid % 64)
    {
      const int m = tid;
      const bool have = m < H || two;
      const size_t g = (size_t)(m < H ? r0 : r1) * H + (m & (H - 1));
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        tmem_ld32(tmem + lane_base + tQ + cc * 32, o);
        tmem_ld_wait();
        if (have && ntiles > 0) {
          uint32_t w[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) w[x] = pack_bf16x2(o[2 * x] * p.scale, o[2 * x + 1] * p.scale);
          uint4* dst = reinterpret_cast<uint4*>(p.dQ + g * D + cc * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(w[4 * x], w[4 * x + 1], w[4 * x + 2], w[4 * x + 3]);
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // the next pair's first dQ MMA overwrites the accumulator
  }
  cp_async_wait_all();
  if (__syncthreads_or(bad) && tid == 0) report_status(p.st, kStatusBounds, 813);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

// =============================================================================================
// launchers
// =============================================================================================
cudaError_t launch_prep(const __nv_bfloat16* dO, const __nv_bfloat16* out, const float* lse, float* Dv, float* lse2,
                        long long n_rows, int D, cudaStream_t stream) {
  long long blocks = (n_rows + 7) / 8;
  if (blocks > 148 * 16) blocks = 148 * 16;
  if (blocks < 1) blocks = 1;
  LaunchScope ls("bwd_prep", stream);
  if (D == 128) return launch_k(bwd_prep_kernel<128>, dim3((unsigned)blocks), dim3(256), 0, stream, true, dO, out, lse, Dv, lse2, n_rows);
  if (D == 64) return launch_k(bwd_prep_kernel<64>, dim3((unsigned)blocks), dim3(256), 0, stream, true, dO, out, lse, Dv, lse2, n_rows);
  return cudaErrorInvalidValue;
}

template <int H, int D>
static cudaError_t launch_full_t(const CUtensorMap& tmQ, const CUtensorMap& tmdO, const CUtensorMap& tmK,
                                 const CUtensorMap& tmV, const BwdParams& p, int sms, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(bwd_dq_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, DqCfg<D>::SMEM);
    cudaFuncSetAttribute(bwd_dkdv_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, KvCfg<D>::SMEM);
    configured = true;
  }
  const int n_dq = p.B * p.tiles_per_batch;
  const int n_kv = p.B * p.kv_tiles * p.n_chunks;
  cudaError_t e;
  {
    LaunchScope ls("bwd_dq", stream);
    e = launch_k(bwd_dq_kernel<H, D>, dim3(n_dq < sms ? n_dq : sms), dim3(NT), DqCfg<D>::SMEM, stream, true, tmQ, tmdO,
                 tmK, tmV, p);
  }
  if (e != cudaSuccess) return e;
  {
    LaunchScope ls("bwd_dkdv", stream);
    e = launch_k(bwd_dkdv_kernel<H, D>, dim3(n_kv < sms ? n_kv : sms), dim3(NT), KvCfg<D>::SMEM, stream, true, tmQ,
                 tmdO, tmK, tmV, p);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_full_bwd(const CUtensorMap& tmQ, const CUtensorMap& tmdO, const CUtensorMap& tmK,
                            const CUtensorMap& tmV, const BwdParams& p, int sms, cudaStream_t stream) {
  if (p.H == 64 && p.D == 128) return launch_full_t<64, 128>(tmQ, tmdO, tmK, tmV, p, sms, stream);
  if (p.H == 16 && p.D == 64) return launch_full_t<16, 64>(tmQ, tmdO, tmK, tmV, p, sms, stream);
  return cudaErrorInvalidValue;
}

template <int H, int D>
static cudaError_t launch_sparse_t(const BwdParams& p, int sms, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(sparse_bwd_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SbCfg<D>::SMEM);
    configured = true;
  }
  const int rows = p.B * p.Lq;
  LaunchScope ls("sparse_bwd", stream);
  const cudaError_t e = launch_k(sparse_bwd_kernel<H, D>, dim3(rows < sms ? rows : sms), dim3(128), SbCfg<D>::SMEM,
                                 stream, true, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_sparse_bwd(const BwdParams& p, int sms, cudaStream_t stream) {
  if (p.H == 64 && p.D == 128 && p.Lq >= 2 && p.S <= PAIR_MAX / 2) {
    // two adjacent rows per CTA over the union of their selections
    static bool configured = false;
    if (!configured) {
      cudaFuncSetAttribute(sparse_bwd_pair_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg<128>::SMEM);
      configured = true;
    }
    const int pairs = p.B * ((p.Lq + 1) / 2);
    LaunchScope ls("sparse_bwd", stream);
    const cudaError_t e = launch_k(sparse_bwd_pair_kernel<128>, dim3(pairs < sms ? pairs : sms), dim3(128),
                                   PairCfg<128>::SMEM, stream, true, p);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  if (p.H == 64 && p.D == 128) return launch_sparse_t<64, 128>(p, sms, stream);
  if (p.H == 16 && p.D == 64) return launch_sparse_t<16, 64>(p, sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace bwd
}  // namespace hs2
