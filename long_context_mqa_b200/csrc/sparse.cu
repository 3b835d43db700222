// Sparse attention of one sparse layer over the full layer's selected tokens (KV Reuse).
//
// One CTA = one query row (b, i) x one split of its index list. For each tile of 128 index
// slots the CTA gathers the 128 selected K rows and V rows ONCE for all H heads (MQA: every
// head reads the same rows) with 16-byte cp.async into 128B-swizzled shared memory, then
//   S = Q K_sel^T            tcgen05, M = 64 rows = the heads (padded to 64), N = 128 keys
//   softmax per head         in-thread: the thread owning a head row holds its 128 logits,
//                            keeps a running (max, sum) across tiles and rescales its O row
//                            in TMEM only when the max grows by more than 2^8
//   O += P V_sel             tcgen05, M = 64 heads, N = d, P (bf16) K-major in shared memory
// TMEM rows of an M = 64 accumulator sit in lanes 0..15 of each 32-lane quarter, so thread
// (warp q, lane l < 16) owns head row 16 q + l. Two CTAs share an SM, so one CTA's gathers
// overlap the other's math. With one split the CTA writes the final bf16 output (and lse); with
// several, every split writes an unnormalised partial and the split that arrives last on the
// row's counter merges them (few query rows, as in decode).
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
  static constexpr int BYTES = OFF_P + P_BYTES + 1024;
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
  __shared__ int s_last;
  __shared__ float wgt[33 * MH];  // merge weights [nsplit][64] and 1/L [64] (nsplit <= 32)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x;  // flattened query row b * Lq + i
  const int b = r / p.Lq;
  const int split = blockIdx.y;
  const int slot0 = split * p.split_slots;
  int slot1 = slot0 + p.split_slots;
  if (slot1 > p.S) slot1 = p.S;
  const int ntiles = (slot1 - slot0 + TILE - 1) / TILE;
  const int32_t* idx_row = p.idx + (size_t)r * p.S;
  const __nv_bfloat16* Kb = p.K + (size_t)b * p.Lk * D;
  const __nv_bfloat16* Vb = p.V + (size_t)b * p.Lk * D;
  const uint32_t tS = 0, tO = 128;
  const int head = warp * 16 + lane;        // the head row this thread owns (lanes 0..15)
  const bool owns = lane < 16 && head < H;  // a real head
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

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

  // thread `tid` gathers key row `tid` of tile t (K tile K-major; the V tile is read MN-major)
  auto gather = [&](int t) {
    const int slot = slot0 + t * TILE + tid;
    int j = -1;
    if (slot < slot1) j = idx_row[slot];
    const bool valid = j >= 0 && j < p.Lk;
    if (j != -1 && !valid) bad = true;
    const __nv_bfloat16* kr = Kb + (size_t)(valid ? j : 0) * D;
    const __nv_bfloat16* vr = Vb + (size_t)(valid ? j : 0) * D;
    const uint32_t kd = smem_u32(sK), vd = smem_u32(sV);
#pragma unroll
    for (int ch = 0; ch < D / 8; ++ch) {
      const uint32_t off = (ch / 8) * (TILE * 128) + sw128_off(tid, ch % 8);
      cp_async_16(kd + off, kr + ch * 8, valid);
      cp_async_16(vd + off, vr + ch * 8, valid);
    }
    cp_async_commit();
    const unsigned m = __ballot_sync(0xffffffffu, valid);
    if (lane == 0) vmask[warp] = m;
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

  for (int t = 0; t < ntiles && ok; ++t) {
    cp_async_wait_all();
    fence_async_smem();
    __syncthreads();
    const bool all_valid = (vmask[0] & vmask[1] & vmask[2] & vmask[3]) == 0xFFFFFFFFu;
    // ---- S = Q K^T
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t IDESC = idesc_bf16(MH, TILE, 0, 0);
      const uint64_t qa = sdesc(smem_u32(sQ), 16, 1024), ka = sdesc(smem_u32(sK), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t a = sdesc_at(qa, (kk / 4) * (MH * 128) + (kk % 4) * 32);
        const uint64_t bk = sdesc_at(ka, (kk / 4) * (TILE * 128) + (kk % 4) * 32);
        umma_bf16(tmem + tS, a, bk, IDESC, kk > 0);
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
    // ---- row max of the valid keys (every thread runs the warp-collective loads)
    float rmax = -INFINITY;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      tmem_ld32(tmem + lane_base + tS + cc * 32, v);
      tmem_ld_wait();
      if (!all_valid) {
        const unsigned mk = vmask[cc];
#pragma unroll
        for (int x = 0; x < 32; ++x) v[x] = (mk >> x) & 1u ? v[x] : -INFINITY;
      }
      rmax = fmaxf(rmax, max32(v));
    }
    const float mt = rmax * c;
    const bool raise = mt > -INFINITY && (m_run == -INFINITY || mt > m_run + RESCALE_SLACK);
    const float alpha = raise ? (m_run == -INFINITY ? 0.f : fast_exp2(m_run - mt)) : 1.f;
    if (raise) m_run = mt;
    l_run *= alpha;
    if (t > 0 && __any_sync(0xffffffffu, raise)) {  // O row *= alpha (warp-collective)
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
    float la = 0.f, lb = 0.f;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      float v[32];
      tmem_ld32(tmem + lane_base + tS + cc * 32, v);
      tmem_ld_wait();
      const unsigned mk = all_valid ? 0xFFFFFFFFu : vmask[cc];
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
      if (lane < 16) {
        const uint32_t blk = smem_u32(sP) + (cc / 2) * (MH * 128);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          st_shared_v4(blk + sw128_off(head, (cc % 2) * 4 + q), pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
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
        umma_bf16(tmem + tO, a, bv, IDESC, (t == 0 && kk == 0) ? 0u : 1u);
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
    if (ok && t + 1 < ntiles) gather(t + 1);  // the single K/V stage is free again
  }
  cp_async_wait_all();
  if (__syncthreads_or(bad) && tid == 0) report_status(p.st, kStatusBounds, 403);
  // ---- epilogue: this thread's O row
  if (ntiles > 0 && ok) {  // block-uniform
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      float o[32];
      tmem_ld32(tmem + lane_base + tO + cc * 32, o);
      tmem_ld_wait();
      if (owns) {
        if (p.nsplit == 1) {
          const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(o[2 * x] * inv, o[2 * x + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)r * H + head) * D + cc * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        } else {
          float4* dst = reinterpret_cast<float4*>(p.opart + (((size_t)r * p.nsplit + split) * H + head) * D + cc * 32);
#pragma unroll
          for (int x = 0; x < 8; ++x) dst[x] = make_float4(o[4 * x], o[4 * x + 1], o[4 * x + 2], o[4 * x + 3]);
        }
      }
    }
  } else if (owns && p.nsplit > 1) {
    float* dst = p.opart + (((size_t)r * p.nsplit + split) * H + head) * D;
    for (int x = 0; x < D; ++x) dst[x] = 0.f;
  }
  if (owns) {
    if (p.nsplit == 1) {
      if (p.lse) p.lse[(size_t)r * H + head] = (m_run + log2f(l_run)) * 0.69314718055994531f;
    } else {
      float* ml = p.mlpart + ((size_t)r * p.nsplit + split) * 2 * H;
      ml[head] = l_run > 0.f ? m_run : -INFINITY;
      ml[H + head] = l_run;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 256); }
  if (p.nsplit > 1) {
    // the split that arrives last on this row's counter merges the row's partials
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&p.counters[r], 1) == p.nsplit - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      const float* mlr = p.mlpart + (size_t)r * p.nsplit * 2 * H;
      if (tid < H) {
        float M = -INFINITY, L = 0.f;
        for (int s2 = 0; s2 < p.nsplit; ++s2)
          if (__ldcg(&mlr[s2 * 2 * H + H + tid]) > 0.f) M = fmaxf(M, __ldcg(&mlr[s2 * 2 * H + tid]));
        for (int s2 = 0; s2 < p.nsplit; ++s2) {
          const float l = __ldcg(&mlr[s2 * 2 * H + H + tid]);
          const float w = l > 0.f ? exp2f(__ldcg(&mlr[s2 * 2 * H + tid]) - M) : 0.f;
          wgt[s2 * MH + tid] = w;
          L += l * w;
        }
        wgt[p.nsplit * MH + tid] = L > 0.f ? 1.f / L : 0.f;
        if (p.lse) p.lse[(size_t)r * H + tid] = (M + log2f(L)) * 0.69314718055994531f;
      }
      __syncthreads();
      // every thread owns EPT float4 columns; a split's loads are all issued before any is used
      const float4* op = reinterpret_cast<const float4*>(p.opart + (size_t)r * p.nsplit * H * D);
      constexpr int EPT_ALL = H * D / 4 / NT;
      constexpr int EPT = EPT_ALL > 8 ? 8 : EPT_ALL;
#pragma unroll 1
      for (int base = 0; base < EPT_ALL; base += EPT) {
        float4 acc[EPT];
#pragma unroll
        for (int q2 = 0; q2 < EPT; ++q2) acc[q2] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s2 = 0; s2 < p.nsplit; ++s2) {
          float4 v4[EPT];
#pragma unroll
          for (int q2 = 0; q2 < EPT; ++q2) v4[q2] = __ldcg(&op[(size_t)s2 * (H * D / 4) + tid + (base + q2) * NT]);
#pragma unroll
          for (int q2 = 0; q2 < EPT; ++q2) {
            const float w = wgt[s2 * MH + (tid + (base + q2) * NT) / (D / 4)];
            acc[q2].x += w * v4[q2].x; acc[q2].y += w * v4[q2].y; acc[q2].z += w * v4[q2].z; acc[q2].w += w * v4[q2].w;
          }
        }
#pragma unroll
        for (int q2 = 0; q2 < EPT; ++q2) {
          const int e = tid + (base + q2) * NT;
          const float inv = wgt[p.nsplit * MH + e / (D / 4)];
          uint2 o2;
          o2.x = pack_bf16x2(acc[q2].x * inv, acc[q2].y * inv);
          o2.y = pack_bf16x2(acc[q2].z * inv, acc[q2].w * inv);
          reinterpret_cast<uint2*>(p.out + (size_t)r * H * D)[e] = o2;
        }
      }
    }
  }
}

size_t sparse_smem_bytes(int H, int D) {
  if (H == 64 && D == 128) return SpLayout<64, 128>::BYTES;
  if (H == 16 && D == 64) return SpLayout<16, 64>::BYTES;
  return 0;
}

template <int H, int D>
static cudaError_t launch_t(const SpParams& p, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(sparse_attn_kernel<H, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SpLayout<H, D>::BYTES);
    configured = true;
  }
  const int rows = p.B * p.Lq;
  if (p.nsplit > 1 && cudaMemsetAsync(p.counters, 0, (size_t)rows * sizeof(int), stream) != cudaSuccess)
    return cudaErrorUnknown;
  LaunchScope ls("sparse_attn", stream);
  sparse_attn_kernel<H, D><<<dim3(rows, p.nsplit), NT, SpLayout<H, D>::BYTES, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_sparse(const SpParams& p, int H, int D, cudaStream_t stream) {
  if (p.nsplit > 32) return cudaErrorInvalidValue;  // merge-weight table holds 32 splits
  if (H == 64 && D == 128) return launch_t<64, 128>(p, stream);
  if (H == 16 && D == 64) return launch_t<16, 64>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sparse
}  // namespace hs2
