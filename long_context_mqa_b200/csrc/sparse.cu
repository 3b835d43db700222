// Sparse attention of one sparse layer over the full layer's selected tokens (KV Reuse).
//
// One CTA = one query row (b, i) x one split of its index list. For each tile of 128 index
// slots the CTA gathers the 128 selected K rows and V rows ONCE for all H heads (MQA: every
// head reads the same rows) with 16-byte cp.async into 128B-swizzled shared memory (an e4m3
// cache: 16-byte loads of 16 codes, widened exactly to bf16 in registers, then stored), then
//   S = Q K_sel^T            tcgen05, M = 64 rows = the heads (padded to 64), N = 128 keys
//   softmax per head         in-thread: the thread owning a head row holds its 128 logits,
//                            keeps a running (max, sum) across tiles and rescales its O row
//                            in TMEM only when the max grows by more than 2^8
//   O += P V_sel             tcgen05, M = 64 heads, N = d, P (bf16) K-major in shared memory
// TMEM rows of an M = 64 accumulator sit in lanes 0..15 of each 32-lane quarter, so thread
// (warp q, lane l < 16) owns head row 16 q + l; lane l + 16 takes over the upper half of that
// row's keys for the softmax. Without splits two CTAs share an SM, so one CTA's gathers overlap
// the other's math. With one split the CTA writes the final bf16 output (and lse). With few query rows
// (decode) a row's index list is split over a cluster of CTAs; head h of the row is merged by
// cluster rank h % n: as soon as its own tiles are done (and every CTA of the cluster has
// started: a cluster barrier arrived at the start, waited on here) each CTA stores its
// unnormalised O rows and per-head (max, sum) into their owners' exchange buffers, and after a
// second cluster barrier each CTA merges its heads from local shared memory. Launched as a programmatic dependent: the prologue overlaps the previous kernel's
// tail and every global read waits for it.
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace sparse {

constexpr int TILE = 128;
constexpr int NT = 128;
constexpr int MH = 64;                 // MMA rows (heads, zero-padded to 64)
constexpr float RESCALE_SLACK = 8.f;   // log2 units

template <int H, int D>
struct SpLayout {
  static constexpr int Q_BYTES = MH * D * 2;     // K-major A operand [64 x D]
  static constexpr int KT_BYTES = TILE * D * 2;  // one gathered K (or V) tile
  static constexpr int P_BYTES = MH * TILE * 2;  // K-major A operand [64 x 128 keys]
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = ((Q_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_V = OFF_K + KT_BYTES;
  static constexpr int OFF_P = OFF_V + KT_BYTES;
  static constexpr int OFF_X = OFF_P + P_BYTES;  // split-merge exchange buffers (clusters only)
  // xO[n][HPR][D] + xm[n][MH] + xl[n][MH] floats, HPR = ceil(H / n) heads per cluster rank
  __host__ __device__ static constexpr int x_bytes(int n) { return n > 1 ? (n * ((H + n - 1) / n) * D + 2 * n * MH) * 4 : 0; }
  __host__ __device__ static constexpr int bytes(int n) { return OFF_X + x_bytes(n) + 1024; }
  static constexpr int max_bytes() {
    int m = bytes(1);
    for (int n = 2; n <= 16; ++n) m = bytes(n) > m ? bytes(n) : m;
    return m;
  }
};

template <int H, int D>
__global__ void __launch_bounds__(NT, 2) sparse_attn_kernel(SpParams p) {
  using Lay = SpLayout<H, D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  uint8_t* sP = smem + Lay::OFF_P;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ unsigned vmask[TILE / 32];
  __shared__ float wgt[17 * MH];  // merge weights [nsplit][heads of this rank] and their 1/L

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x;  // flattened query row b * Lq + i
  const int b = r / p.Lq;
  const int split = blockIdx.y;
  const int slot0 = split * p.split_slots;
  int slot1 = slot0 + p.split_slots;
  if (slot1 > p.S) slot1 = p.S;
  const int ntiles = (slot1 - slot0 + TILE - 1) / TILE;
  const int32_t* idx_row = p.idx + (size_t)r * p.S;
  // the rows of this row's sequence (contiguous cache) or the page pools (paged cache)
  const __nv_bfloat16* Kb = p.ptab ? p.K : p.K + (size_t)b * p.Lk * D;
  const __nv_bfloat16* Vb = p.ptab ? p.V : p.V + (size_t)b * p.Lk * D;
  const uint32_t tS = 0, tO = 128;
  const int prow = warp * 16 + (lane & 15);  // the row this lane's pair works on
  const int head = warp * 16 + lane;         // the head row this thread owns (lanes 0..15)
  const bool owns = lane < 16 && head < H;   // a real head, written out by this lane
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  // every input may come from the kernels before this one on the stream
  griddep_wait();
  griddep_launch_dependents();
  // first half of the cluster barrier that makes the other CTAs' shared memory safe to write
  // (every CTA of the cluster has started); its wait comes just before the first remote store
  if (p.nsplit > 1) cluster_arrive();
  // ---- query -> shared (K-major, 128B swizzle): rows 0..H-1 by cp.async, padding rows zero
  {
    const __nv_bfloat16* q = p.Q + (size_t)r * H * D;
    for (int c = tid; c < MH * D / 8; c += NT) {
      const int row = c / (D / 8), ch = c % (D / 8);
      const uint32_t dst = smem_u32(sQ) + (ch / 8) * (MH * 128) + sw128_off(row, ch % 8);
      if (row < H) cp_async_16(dst, q + row * D + ch * 8, true);
      else st_shared_v4(dst, 0u, 0u, 0u, 0u);
    }
  }
  if (tid == 0) { mbar_init(&mma_bar, 1); fence_mbar_init(); }
  if (warp == 0) { tmem_alloc(&tmem_base, 256); tmem_relinquish(); }
  bool bad = false;

  // gathers the key rows of tile t (K tile K-major; the V tile is read MN-major). Thread `tid`
  // reads the index of row `tid`; the copies are coalesced: LPR consecutive lanes fetch the
  // 16-byte chunks of one row (a whole row per group of lanes, RPS rows per warp step), the
  // row's index passed by shuffle from the lane that read it.
  auto gather = [&](int t) {
    constexpr int LPR = D * 2 / 16, RPS = 32 / LPR;
    const int slot = slot0 + t * TILE + tid;
    int j = -1;
    if (slot < slot1) j = idx_row[slot];
    bool valid = j >= 0 && j < p.Lk;
    // the row of token j: row j of the sequence's cache, or (paged) row j % 128 of its page
    long long krow = -1;
    if (valid) {
      if (p.ptab) {
        const int pg = __ldg(p.ptab + (size_t)b * p.max_pages + (j >> 7));
        valid = pg >= 0 && pg < p.n_pages;
        krow = valid ? (long long)pg * 128 + (j & 127) : -1;
      } else {
        krow = j;
      }
    }
    if (j != -1 && !valid) bad = true;
    const unsigned m = __ballot_sync(0xffffffffu, valid);
    if (lane == 0) vmask[warp] = m;
    const uint32_t kd = smem_u32(sK), vd = smem_u32(sV);
    if (p.K8) {
      // e4m3 cache: rows of D bytes, LPR8 lanes per row, 16 codes per lane, widened exactly to
      // bf16 in registers (all loads issued before the first conversion)
      constexpr int LPR8 = D / 16, RPS8 = 32 / LPR8;
      const int sub8 = lane / LPR8, ch8 = lane % LPR8;
      const uint8_t* K8b = p.ptab ? p.K8 : p.K8 + (size_t)b * p.Lk * D;
      const uint8_t* V8b = p.ptab ? p.V8 : p.V8 + (size_t)b * p.Lk * D;
      uint4 xk[32 / RPS8], xv[32 / RPS8];
#pragma unroll
      for (int it = 0; it < 32 / RPS8; ++it) {
        const long long kr = __shfl_sync(0xffffffffu, krow, it * RPS8 + sub8);
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        xk[it] = kr >= 0 ? __ldg(reinterpret_cast<const uint4*>(K8b + (size_t)kr * D) + ch8) : z;
        xv[it] = kr >= 0 ? __ldg(reinterpret_cast<const uint4*>(V8b + (size_t)kr * D) + ch8) : z;
      }
      auto put = [&](uint32_t base, int rr, const uint4& x) {
        const uint32_t o = base + (ch8 / 4) * (TILE * 128);
        st_shared_v4(o + sw128_off(rr, (2 * ch8) % 8), e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.x)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.x >> 16)), e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.y)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.y >> 16)));
        st_shared_v4(o + sw128_off(rr, (2 * ch8 + 1) % 8), e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.z)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.z >> 16)), e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.w)),
                     e4m3_f16x2_to_bf16x2(e4m3x2_to_f16x2(x.w >> 16)));
      };
#pragma unroll
      for (int it = 0; it < 32 / RPS8; ++it) {
        const int rr = warp * 32 + it * RPS8 + sub8;
        put(kd, rr, xk[it]);
        put(vd, rr, xv[it]);
      }
      cp_async_commit();  // (an empty group: the wait before the MMAs stays uniform)
      return;
    }
    const int sub = lane / LPR, ch = lane % LPR;
#pragma unroll
    for (int it = 0; it < 32 / RPS; ++it) {
      const int rr = it * RPS + sub;  // row within this warp's 32
      const long long kr = __shfl_sync(0xffffffffu, krow, rr);
      const uint32_t off = (ch / 8) * (TILE * 128) + sw128_off(warp * 32 + rr, ch % 8);
      const size_t src = (size_t)(kr >= 0 ? kr : 0) * D + ch * 8;
      cp_async_16(kd + off, Kb + src, kr >= 0);
      cp_async_16(vd + off, Vb + src, kr >= 0);
    }
    cp_async_commit();
  };

  const float c = p.c;
  float m_run = -INFINITY, l_run = 0.f;
  uint32_t phase = 0;
  bool ok = true;
  if (ntiles > 0) gather(0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;

  bool any_pv = false;  // a PV has written O (block-uniform)
  for (int t = 0; t < ntiles && ok; ++t) {
    cp_async_wait_all();
    fence_async_smem();
    __syncthreads();
    const bool all_valid = (vmask[0] & vmask[1] & vmask[2] & vmask[3]) == 0xFFFFFFFFu;
    if ((vmask[0] | vmask[1] | vmask[2] | vmask[3]) == 0u) {
      // no valid slot in the tile (a list's -1 tail): nothing to add. Every thread has read the
      // masks before the next gather rewrites them.
      __syncthreads();
      if (t + 1 < ntiles) gather(t + 1);
      continue;
    }
    // ---- S = Q K^T
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t IDESC = idesc_bf16(MH, TILE, 0, 0);
      const uint64_t qa = sdesc(smem_u32(sQ), 16, 1024), ka = sdesc(smem_u32(sK), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t a = sdesc_at(qa, (kk / 4) * (MH * 128) + (kk % 4) * 32);
        const uint64_t bk = sdesc_at(ka, (kk / 4) * (TILE * 128) + (kk % 4) * 32);
        umma_ss(tmem + tS, a, bk, IDESC, kk > 0);
      }
      umma_commit(&mma_bar);
    }
    {
      bool w_ok = true;
      if (tid == 0) w_ok = mbar_wait(&mma_bar, phase, p.wait_ns);
      if (!__syncthreads_and(w_ok)) { if (tid == 0) report_status(p.st, kStatusTimeout, 401); ok = false; }
    }
    phase ^= 1;
    if (!ok) break;
    tc_fence_after();
    // ---- the row's 128 logits (warp-collective loads, one wait). The head rows sit in the first
    // 16 lanes of each quarter; lane l reads keys 0..63 of row l and lane l + 16 keys 64..127 of
    // the same row, so every lane exponentiates 64 keys. Both lanes of a pair keep the same
    // running max.
    const bool upper = lane >= 16;
    float sv[2][32];
    tmem_ld16x2_32<64>(tmem + lane_base + tS, sv[0]);       // keys 0..31 | 64..95
    tmem_ld16x2_32<64>(tmem + lane_base + tS + 32, sv[1]);  // keys 32..63 | 96..127
    tmem_ld_wait();
    float rmax = -INFINITY;
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      if (!all_valid) {
        const unsigned mk = vmask[(upper ? 2 : 0) + h2];
#pragma unroll
        for (int x = 0; x < 32; ++x) sv[h2][x] = (mk >> x) & 1u ? sv[h2][x] : -INFINITY;
      }
      rmax = fmaxf(rmax, max32(sv[h2]));
    }
    rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 16));
    const float mt = rmax * c;
    const bool raise = mt > -INFINITY && (m_run == -INFINITY || mt > m_run + RESCALE_SLACK);
    const float alpha = raise ? (m_run == -INFINITY ? 0.f : fast_exp2(m_run - mt)) : 1.f;
    if (raise) m_run = mt;
    l_run *= alpha;
    if (any_pv && __any_sync(0xffffffffu, raise)) {  // O row *= alpha (warp-collective)
#pragma unroll
      for (int cc = 0; cc < D / 16; ++cc) {
        float o[16];
        tmem_ld16(tmem + lane_base + tO + cc * 16, o);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 16; ++x) o[x] *= alpha;
        tmem_st16(tmem + lane_base + tO + cc * 16, o);
      }
      tmem_st_wait();
    }
    // ---- probabilities -> P row (K-major: row = head, K = the 128 keys)
    const float negm = m_run == -INFINITY ? 0.f : -m_run;
    float la = 0.f, lb = 0.f;  // this lane's half of the row sum (l_run is the half's running sum)
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const float* v = sv[h2];
      const unsigned mk = all_valid ? 0xFFFFFFFFu : vmask[(upper ? 2 : 0) + h2];
      uint32_t pk[16];
#pragma unroll
      for (int x = 0; x < 32; x += 2) {
        float e0, e1;
        ffma2(e0, e1, v[x], v[x + 1], c, c, negm, negm);
        const float p0 = (mk >> x) & 1u ? fast_exp2(e0) : 0.f;
        const float p1 = (mk >> (x + 1)) & 1u ? fast_exp2(e1) : 0.f;
        fadd2(la, lb, la, lb, p0, p1);
        pk[x / 2] = pack_bf16x2(p0, p1);
      }
      {  // keys 0..63 of the row in the first 128-byte block, keys 64..127 in the second
        const uint32_t blk = smem_u32(sP) + (upper ? MH * 128 : 0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(blk + sw128_off(prow, h2 * 4 + q), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
      }
    }
    l_run += la + lb;
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    // ---- O += P V
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t IDESC = idesc_bf16(MH, D, 0, 1);
      const uint64_t pa = sdesc(smem_u32(sP), 16, 1024), va = sdesc(smem_u32(sV), TILE * 128, 1024);
#pragma unroll
      for (int kk = 0; kk < TILE / 16; ++kk) {
        const uint64_t a = sdesc_at(pa, (kk / 4) * (MH * 128) + (kk % 4) * 32);
        const uint64_t bv = sdesc_at(va, kk * 2048);
        umma_ss(tmem + tO, a, bv, IDESC, (!any_pv && kk == 0) ? 0u : 1u);
      }
      umma_commit(&mma_bar);
    }
    {
      bool w_ok = true;
      if (tid == 0) w_ok = mbar_wait(&mma_bar, phase, p.wait_ns);
      if (!__syncthreads_and(w_ok)) { if (tid == 0) report_status(p.st, kStatusTimeout, 402); ok = false; }
    }
    phase ^= 1;
    tc_fence_after();
    any_pv = true;
    if (ok && t + 1 < ntiles) gather(t + 1);  // the single K/V stage is free again
  }
  cp_async_wait_all();
  if (__syncthreads_or(bad) && tid == 0) report_status(p.st, kStatusBounds, 403);
  // ---- epilogue
  const bool have = any_pv && ok;  // block-uniform
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);  // the row's sum: both halves
  // lane l < 16 holds columns 32 i .. 32 i + 31 of head row prow, lane l + 16 the same columns
  // shifted by D / 2 (i < D / 64)
  const int cbase = lane >= 16 ? D / 2 : 0;
  if (p.nsplit == 1) {
    if (have) {
      const float inv = l_run > 0.f ? p.oscale / l_run : 0.f;
#pragma unroll
      for (int i = 0; i < D / 64; ++i) {
        float o[32];
        tmem_ld16x2_32<D / 2>(tmem + lane_base + tO + i * 32, o);
        tmem_ld_wait();
        if (prow < H) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(o[2 * x] * inv, o[2 * x + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)r * H + prow) * D + cbase + i * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
    } else if (ok && prow < H) {  // the row selected nothing: zeros
      uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)r * H + prow) * D + cbase);
#pragma unroll
      for (int x = 0; x < D / 16; ++x) dst[x] = make_uint4(0u, 0u, 0u, 0u);
    }
    if (owns && p.lse) p.lse[(size_t)r * H + head] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    tc_fence_before();
    __syncthreads();
    if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 256); }
    return;
  }
  // cluster merge. Exchange buffers in their own shared-memory region of every CTA:
  //   xO[s][k][D]  O row of head rank + k*n from split s      (HPR = ceil(H / n) heads per rank)
  //   xm[s][MH], xl[s][MH]  split s's max (log2 units) and sum per head
  const int n = p.nsplit;
  const uint32_t rank = cluster_ctarank();
  const int HPR = (H + n - 1) / n;
  float* xO = reinterpret_cast<float*>(smem + Lay::OFF_X);
  float* xm = xO + (size_t)n * HPR * D;
  float* xl = xm + n * MH;
  {
    // this CTA's O rows (unnormalised; both lanes of a pair hold half a row), one TMEM wait,
    // while the cluster barrier completes
    float o[D / 64][32];
    if (have) {
#pragma unroll
      for (int i = 0; i < D / 64; ++i) tmem_ld16x2_32<D / 2>(tmem + lane_base + tO + i * 32, o[i]);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int i = 0; i < D / 64; ++i)
#pragma unroll
        for (int x = 0; x < 32; ++x) o[i][x] = 0.f;
    }
    cluster_wait();  // every CTA of the cluster has started: its shared memory can be written
    const int owner = prow % n, k = prow / n;
    if (prow < H) {
      const uint32_t o_dst = dsmem_addr(smem_u32(xO + ((size_t)split * HPR + k) * D + cbase), owner);
#pragma unroll
      for (int i = 0; i < D / 64; ++i)
#pragma unroll
        for (int x = 0; x < 8; ++x)
          st_dsmem_v4(o_dst + (i * 32 + 4 * x) * 4, o[i][4 * x], o[i][4 * x + 1], o[i][4 * x + 2], o[i][4 * x + 3]);
    }
    if (owns) {
      const float mv = l_run > 0.f && have ? m_run : -INFINITY, lv = have ? l_run : 0.f;
      // only the owner reads head `head`'s (max, sum)
      const uint32_t m_loc = smem_u32(xm + split * MH + head), l_loc = smem_u32(xl + split * MH + head);
      st_dsmem_f32(dsmem_addr(m_loc, (uint32_t)owner), mv);
      st_dsmem_f32(dsmem_addr(l_loc, (uint32_t)owner), lv);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 256); }
  cluster_sync_all();  // all partials have landed; nothing reads another CTA's memory after this
  // merge weights of this rank's heads: a group of 16 lanes per head (lane s = split s), the
  // max and the sum by shuffles within the group; every lane of a warp takes the same number
  // of steps, so the shuffles are warp-uniform
  {
    const int s = tid & 15;
    for (int k0 = 0; k0 < HPR; k0 += NT / 16) {
      const int k = k0 + (tid >> 4);
      const int h = (int)rank + k * n;
      const bool hv = k < HPR && h < H;
      const bool on = hv && s < n;
      const float lx = on ? xl[s * MH + h] : 0.f;
      const float mx = lx > 0.f ? xm[s * MH + h] : -INFINITY;
      if (!p.gate) {
        float M = mx;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        const float w = lx > 0.f ? exp2f(mx - M) : 0.f;
        float L = lx * w;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
        if (on) wgt[s * MH + k] = w;
        if (hv && s == 0) {
          wgt[16 * MH + k] = L > 0.f ? p.oscale / L : 0.f;
          if (p.lse) p.lse[(size_t)r * H + h] = (M + log2f(L)) * 0.69314718055994531f;
        }
      } else {
        // two branches, each its own softmax (splits below branch_split: the blocks; the rest:
        // the window), mixed by the gate: the weights carry each branch's normalisation and share
        const bool br = s >= p.branch_split;
        float M0 = br ? -INFINITY : mx, M1 = br ? mx : -INFINITY;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          M0 = fmaxf(M0, __shfl_xor_sync(0xffffffffu, M0, o));
          M1 = fmaxf(M1, __shfl_xor_sync(0xffffffffu, M1, o));
        }
        const float w = lx > 0.f ? exp2f(mx - (br ? M1 : M0)) : 0.f;
        float L0 = br ? 0.f : lx * w, L1 = br ? lx * w : 0.f;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) {
          L0 += __shfl_xor_sync(0xffffffffu, L0, o);
          L1 += __shfl_xor_sync(0xffffffffu, L1, o);
        }
        const float g = hv ? p.gate[(size_t)r * H + h] : 0.f;
        const float f0 = L0 > 0.f ? g / L0 : 0.f, f1 = L1 > 0.f ? (1.f - g) / L1 : 0.f;
        if (on) wgt[s * MH + k] = w * (br ? f1 : f0);
        if (hv && s == 0) wgt[16 * MH + k] = p.oscale;
      }
    }
  }
  __syncthreads();
  // this rank's heads, 4 columns per thread per step
  for (int e4 = tid; e4 < HPR * D / 4; e4 += NT) {
    const int k = e4 / (D / 4), d4 = e4 % (D / 4);
    const int h = (int)rank + k * n;
    if (h >= H) continue;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int s2 = 0; s2 < n; ++s2) {
      const float w = wgt[s2 * MH + k];
      const float4 v4 = reinterpret_cast<const float4*>(xO + ((size_t)s2 * HPR + k) * D)[d4];
      acc.x += w * v4.x; acc.y += w * v4.y; acc.z += w * v4.z; acc.w += w * v4.w;
    }
    const float inv = wgt[16 * MH + k];
    uint2 o2;
    o2.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    o2.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(p.out + ((size_t)r * H + h) * D)[d4] = o2;
  }
}


size_t sparse_smem_bytes(int H, int D, int nsplit) {
  if (H == 64 && D == 128) return SpLayout<64, 128>::bytes(nsplit);
  if (H == 16 && D == 64) return SpLayout<16, 64>::bytes(nsplit);
  return 0;
}

template <int H, int D>
static cudaError_t launch_t(const SpParams& p, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(sparse_attn_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         SpLayout<H, D>::max_bytes());
    cudaFuncSetAttribute(sparse_attn_kernel<H, D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    configured = true;
  }
  const int rows = p.B * p.Lq;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(rows, p.nsplit);
  cfg.blockDim = dim3(NT);
  cfg.dynamicSmemBytes = SpLayout<H, D>::bytes(p.nsplit);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;  // the splits of one row form a cluster
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = p.nsplit;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = p.nsplit > 1 ? attr : attr + 1;
  cfg.numAttrs = p.nsplit > 1 ? 2 : 1;
  LaunchScope ls("sparse_attn", stream);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, sparse_attn_kernel<H, D>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_sparse(const SpParams& p, int H, int D, cudaStream_t stream) {
  if (p.nsplit < 1 || p.nsplit > 16) return cudaErrorInvalidValue;  // merge table and cluster size
  // the gated branches merge across the cluster: at least one split on each side of the boundary
  if (p.gate && (p.nsplit < 2 || p.branch_split < 1 || p.branch_split >= p.nsplit || p.lse))
    return cudaErrorInvalidValue;
  if (H == 64 && D == 128) return launch_t<64, 128>(p, stream);
  if (H == 16 && D == 64) return launch_t<16, 64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sparse
}  // namespace hs2
