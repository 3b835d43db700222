// Sparse attention of one sparse layer over the full layer's selected tokens (KV Reuse).
//
// One CTA = one query row (b, i) x one split of its index list. For each tile of 128 index
// slots the CTA gathers the 128 selected K rows and V rows ONCE for all H heads (MQA: every
// head reads the same rows) with 16-byte cp.async into 128B-swizzled shared memory, then
//   S^T = K_sel Q^T          tcgen05, M = 128 keys (TMEM lanes), N = H heads
//   online softmax per head  (tile max through a transposed shared-memory pass; the running
//                             max is only raised when a tile exceeds it by more than 2^8,
//                             so O^T is rarely rescaled)
//   O^T += V_sel^T P^T       tcgen05, M = d, N = 64 (heads padded to 64), P^T MN-major bf16
// With several tiles per CTA, the gathers of tile t+1 overlap the math of tile t (2 stages);
// with one tile per CTA (few query rows: decode) a single stage keeps two CTAs per SM. With one
// split the CTA writes the final bf16 output (and lse); with several, every split writes an
// unnormalised partial, and the split that arrives last on the row's counter merges them.
// 128 threads; thread r owns key row r of the tile (TMEM lane r) and, for O^T, output
// column d = r (d = 128) or the M=64 lane layout (d = 64).
#include "decode.h"
#include "host_util.h"
#include "tc.cuh"

namespace hs2 {
namespace sparse {

constexpr int TILE = 128;
constexpr int NT = 128;
constexpr float RESCALE_SLACK = 8.f;  // log2 units

template <int H, int D, int STAGES>
struct SpLayout {
  static constexpr int HP = 64;                       // heads padded for the PV MMA
  static constexpr int Q_BYTES = H * D * 2;           // K-major B operand, H rows
  static constexpr int KT_BYTES = TILE * D * 2;
  static constexpr int X_BYTES = TILE * H * 4;          // transpose buffer, XOR-swizzled columns
  static constexpr int P_BYTES = TILE * HP * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = ((Q_BYTES + 1023) / 1024) * 1024;
  static constexpr int OFF_V = OFF_K + STAGES * KT_BYTES;
  static constexpr int OFF_P = OFF_V + STAGES * KT_BYTES;
  // one stage: the K tile is dead once S^T is in TMEM, so the transpose buffer reuses it;
  // two stages: it shares the P^T buffer (P^T is written after the transpose is read)
  static constexpr int XP_BYTES = STAGES == 1 ? P_BYTES : (X_BYTES > P_BYTES ? X_BYTES : P_BYTES);
  static constexpr int OFF_X = STAGES == 1 ? OFF_K : OFF_P;
  static_assert(STAGES == 2 || X_BYTES <= KT_BYTES, "transpose buffer must fit the K tile");
  static constexpr int BYTES = OFF_P + ((XP_BYTES + 1023) / 1024) * 1024 + 1024;
};
// element (row, h) of the transpose buffer; the XOR keeps both access patterns conflict-free
template <int H>
__device__ __forceinline__ int xidx(int row, int h) {
  return row * H + (h ^ (row & ((H < 32 ? H : 32) - 1)));
}

template <int H, int D, int STAGES>
__global__ void __launch_bounds__(NT, 1) sparse_attn_kernel(SpParams p) {
  using Lay = SpLayout<H, D, STAGES>;
  constexpr int HP = Lay::HP;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t* sQ = smem + Lay::OFF_Q;
  uint8_t* sK = smem + Lay::OFF_K;
  uint8_t* sV = smem + Lay::OFF_V;
  float* sX = (float*)(smem + Lay::OFF_X);
  uint8_t* sP = smem + Lay::OFF_P;
  __shared__ __align__(8) uint64_t mma_bar;
  __shared__ uint32_t tmem_base;
  __shared__ float sM[H], sAlpha[H], sL[H];
  __shared__ int s_rescale;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = blockIdx.x;                   // flattened query row b * Lq + i
  const int b = r / p.Lq;
  const int split = blockIdx.y;
  const int slot0 = split * p.split_slots;
  int slot1 = slot0 + p.split_slots;
  if (slot1 > p.S) slot1 = p.S;
  const int ntiles = (slot1 - slot0 + TILE - 1) / TILE;
  const int32_t* idx_row = p.idx + (size_t)r * p.S;
  const __nv_bfloat16* Kb = p.K + (size_t)b * p.Lk * D;
  const __nv_bfloat16* Vb = p.V + (size_t)b * p.Lk * D;
  const uint32_t tS = 0, tO = 64;

  // ---- query -> shared (K-major, 128B swizzle) by cp.async, in flight with tile 0's gather
  {
    const __nv_bfloat16* q = p.Q + (size_t)r * H * D;
    for (int c = tid; c < H * D / 8; c += NT) {
      const int row = c / (D / 8), ch = c % (D / 8);
      cp_async_16(smem_u32(sQ) + (ch / 8) * (H * 128) + sw128_off(row, ch % 8), q + row * D + ch * 8, true);
    }
  }
  if (tid < H) { sM[tid] = -INFINITY; sAlpha[tid] = 1.f; }
  if (tid == 0) { mbar_init(&mma_bar, 1); fence_mbar_init(); s_rescale = 0; }
  bool bad = false;
  if (warp == 0) { tmem_alloc(&tmem_base, 128); tmem_relinquish(); }

  // gather issue: thread `tid` copies key row `tid` of tile `t` into stage `buf`
  auto gather = [&](int t, int buf) -> bool {
    const int slot = slot0 + t * TILE + tid;
    int j = -1;
    if (slot < slot1) j = idx_row[slot];
    bool valid = j >= 0 && j < p.Lk;
    if (j != -1 && !valid) bad = true;
    const __nv_bfloat16* kr = Kb + (size_t)(valid ? j : 0) * D;
    const __nv_bfloat16* vr = Vb + (size_t)(valid ? j : 0) * D;
    const uint32_t kd = smem_u32(sK + buf * Lay::KT_BYTES), vd = smem_u32(sV + buf * Lay::KT_BYTES);
#pragma unroll
    for (int ch = 0; ch < D / 8; ++ch) {
      const uint32_t off = (ch / 8) * (TILE * 128) + sw128_off(tid, ch % 8);
      cp_async_16(kd + off, kr + ch * 8, valid);
      cp_async_16(vd + off, vr + ch * 8, valid);
    }
    cp_async_commit();
    return valid;
  };

  bool valid_cur = ntiles > 0 ? gather(0, 0) : false;
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  const float c = p.c;
  float lsum[H];
#pragma unroll
  for (int h = 0; h < H; ++h) lsum[h] = 0.f;
  uint32_t phase = 0;
  bool ok = true;
  const int quarter = warp & 3;

  for (int t = 0; t < ntiles && ok; ++t) {
    const int buf = STAGES == 2 ? (t & 1) : 0;
    bool valid_next = false;
    if (STAGES == 2 && t + 1 < ntiles) {
      valid_next = gather(t + 1, buf ^ 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      cp_async_wait_all();
    }
    fence_async_smem();
    __syncthreads();
    // ---- S^T = K_sel Q^T
    if (tid == 0) {
      tc_fence_after();
      constexpr uint32_t IDESC = idesc_bf16(128, H, 0, 0);
      const uint32_t ka = smem_u32(sK + buf * Lay::KT_BYTES), qa = smem_u32(sQ);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint64_t a = sdesc(ka + (kk / 4) * (TILE * 128) + (kk % 4) * 32, 16, 1024);
        const uint64_t bq = sdesc(qa + (kk / 4) * (H * 128) + (kk % 4) * 32, 16, 1024);
        umma_bf16(tmem + tS, a, bq, IDESC, kk > 0);
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
    float x[H];
#pragma unroll
    for (int cc = 0; cc < (H + 15) / 16; ++cc) {
      float tmp[16];
      tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + tS + cc * 16, tmp);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        if (cc * 16 + e < H) x[cc * 16 + e] = tmp[e];
    }
    tmem_ld_wait();
    const int row = quarter * 32 + lane;  // == tid
#pragma unroll
    for (int h = 0; h < H; ++h) {
      x[h] = valid_cur ? x[h] * c : -INFINITY;
      sX[xidx<H>(row, h)] = x[h];
    }
    __syncthreads();
    // ---- per-head tile max: TPH threads per head
    {
      constexpr int TPH = NT / H;             // 2 (H = 64) or 8 (H = 16)
      constexpr int ROWS = TILE / TPH;
      const int h = tid / TPH, part = tid % TPH;
      float mx = -INFINITY;
      for (int q2 = 0; q2 < ROWS; ++q2) mx = fmaxf(mx, sX[xidx<H>(part * ROWS + q2, h)]);
#pragma unroll
      for (int o = 1; o < TPH; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (part == 0) {
        const float mold = sM[h];
        float alpha = 1.f;
        if (mx > -INFINITY && (mold == -INFINITY || mx > mold + RESCALE_SLACK)) {
          alpha = mold == -INFINITY ? 0.f : fast_exp2(mold - mx);
          sM[h] = mx;
          s_rescale = 1;
        }
        sAlpha[h] = alpha;
      }
    }
    __syncthreads();
    const bool rescale = s_rescale != 0;
    // ---- probabilities, running sums, P^T row
    uint32_t pk[HP / 2];
#pragma unroll
    for (int i2 = 0; i2 < HP / 2; ++i2) pk[i2] = 0u;
#pragma unroll
    for (int h = 0; h < H; h += 2) {
      const float p0 = valid_cur ? fast_exp2(x[h] - sM[h]) : 0.f;
      const float p1 = valid_cur ? fast_exp2(x[h + 1] - sM[h + 1]) : 0.f;
      lsum[h] = rescale ? fmaf(lsum[h], sAlpha[h], p0) : lsum[h] + p0;
      lsum[h + 1] = rescale ? fmaf(lsum[h + 1], sAlpha[h + 1], p1) : lsum[h + 1] + p1;
      pk[h / 2] = pack_bf16x2(p0, p1);
    }
    if (rescale && t > 0) {
      // O^T (lane = output column d, column h = head) *= alpha_h; warp-collective, every lane
      {
        float o[HP];
#pragma unroll
        for (int cc = 0; cc < HP / 16; ++cc) {
          float tmp[16];
          tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + tO + cc * 16, tmp);
#pragma unroll
          for (int e = 0; e < 16; ++e) o[cc * 16 + e] = tmp[e];
        }
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < HP / 16; ++cc) {
          float tmp[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) tmp[e] = (cc * 16 + e < H) ? o[cc * 16 + e] * sAlpha[cc * 16 + e] : 0.f;
          tmem_st16(tmem + ((uint32_t)(quarter * 32) << 16) + tO + cc * 16, tmp);
        }
        tmem_st_wait();
      }
    }
    // sX reads are complete (barrier above) -> P^T may overwrite it (two stages share it)
    {
      const uint32_t prow = smem_u32(sP);
#pragma unroll
      for (int ch = 0; ch < HP / 8; ++ch)
        st_shared_v4(prow + sw128_off(row, ch), pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      s_rescale = 0;
      tc_fence_after();
      constexpr uint32_t IDESC = idesc_bf16(D, HP, 1, 1);
      const uint32_t va = smem_u32(sV + buf * Lay::KT_BYTES), pa = smem_u32(sP);
#pragma unroll
      for (int kk = 0; kk < TILE / 16; ++kk) {
        const uint64_t a = sdesc(va + kk * 2048, TILE * 128, 1024);
        const uint64_t bb = sdesc(pa + kk * 2048, TILE * 128, 1024);
        umma_bf16(tmem + tO, a, bb, IDESC, (t == 0 && kk == 0) ? 0u : 1u);
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
    if (STAGES == 1 && t + 1 < ntiles && ok) {  // the only stage is free again
      valid_next = gather(t + 1, 0);
      fence_async_smem();
    }
    valid_cur = valid_next;
  }
  cp_async_wait_all();
  // ---- row sums across the 128 key lanes
#pragma unroll
  for (int h = 0; h < H; ++h) sX[xidx<H>(tid, h)] = lsum[h];
  __syncthreads();
  if (tid < H) {
    float s = 0.f;
    for (int q2 = 0; q2 < TILE; ++q2) s += sX[xidx<H>(q2, tid)];
    sL[tid] = s;
  }
  __syncthreads();
  if (__syncthreads_or(bad) && tid == 0) report_status(p.st, kStatusBounds, 403);
  // ---- O^T -> output (lane = d)
  const bool has_row = (D == 128) || (lane < 16);
  const int d = (D == 128) ? tid : quarter * 16 + lane;
  if (ntiles > 0 && ok) {  // block-uniform
    float o[HP];
#pragma unroll
    for (int cc = 0; cc < HP / 16; ++cc) {
      float tmp[16];
      tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + tO + cc * 16, tmp);
#pragma unroll
      for (int e = 0; e < 16; ++e) o[cc * 16 + e] = tmp[e];
    }
    tmem_ld_wait();
    if (!has_row) {
    } else if (p.nsplit == 1) {
#pragma unroll
      for (int h = 0; h < H; ++h) {
        const float L = sL[h];
        p.out[((size_t)r * H + h) * D + d] = __float2bfloat16_rn(L > 0.f ? o[h] / L : 0.f);
      }
    } else {
      float* dst = p.opart + ((size_t)r * p.nsplit + split) * H * D;
#pragma unroll
      for (int h = 0; h < H; ++h) dst[h * D + d] = o[h];
    }
  } else if (has_row && p.nsplit > 1) {
    float* dst = p.opart + ((size_t)r * p.nsplit + split) * H * D;
    for (int h = 0; h < H; ++h) dst[h * D + d] = 0.f;
  }
  if (tid < H) {
    if (p.nsplit == 1) {
      if (p.lse) p.lse[(size_t)r * H + tid] = (sM[tid] + log2f(sL[tid])) * 0.69314718055994531f;
    } else {
      float* ml = p.mlpart + ((size_t)r * p.nsplit + split) * 2 * H;
      ml[tid] = sM[tid];
      ml[H + tid] = sL[tid];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) { tc_fence_after(); tmem_dealloc(tmem, 128); }
  if (p.nsplit > 1) {
    // the split that arrives last on this row's counter merges the row's partials
    __shared__ int s_last;
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&p.counters[r], 1) == p.nsplit - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      float* wgt = sX;  // [nsplit][H] merge weights, then [H] 1 / L
      const float* mlr = p.mlpart + (size_t)r * p.nsplit * 2 * H;
      if (tid < H) {
        float M = -INFINITY, L = 0.f;
        for (int s2 = 0; s2 < p.nsplit; ++s2)
          if (mlr[s2 * 2 * H + H + tid] > 0.f) M = fmaxf(M, mlr[s2 * 2 * H + tid]);
        for (int s2 = 0; s2 < p.nsplit; ++s2) {
          const float l = mlr[s2 * 2 * H + H + tid];
          const float w = l > 0.f ? exp2f(mlr[s2 * 2 * H + tid] - M) : 0.f;
          wgt[s2 * H + tid] = w;
          L += l * w;
        }
        wgt[p.nsplit * H + tid] = L > 0.f ? 1.f / L : 0.f;
        if (p.lse) p.lse[(size_t)r * H + tid] = (M + log2f(L)) * 0.69314718055994531f;
      }
      __syncthreads();
      const float4* op = reinterpret_cast<const float4*>(p.opart + (size_t)r * p.nsplit * H * D);
      for (int e = tid; e < H * D / 4; e += NT) {
        const int h = e / (D / 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s2 = 0; s2 < p.nsplit; ++s2) {
          const float w = wgt[s2 * H + h];
          const float4 v4 = op[(size_t)s2 * (H * D / 4) + e];
          acc.x += w * v4.x; acc.y += w * v4.y; acc.z += w * v4.z; acc.w += w * v4.w;
        }
        const float inv = wgt[p.nsplit * H + h];
        uint2 o2;
        o2.x = pack_bf16x2(acc.x * inv, acc.y * inv);
        o2.y = pack_bf16x2(acc.z * inv, acc.w * inv);
        reinterpret_cast<uint2*>(p.out + (size_t)r * H * D)[e] = o2;
      }
    }
  }
}

size_t sparse_smem_bytes(int H, int D) {
  if (H == 64 && D == 128) return SpLayout<64, 128, 2>::BYTES;
  if (H == 16 && D == 64) return SpLayout<16, 64, 2>::BYTES;
  return 0;
}

template <int H, int D, int STAGES>
static cudaError_t launch_t(const SpParams& p, cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(sparse_attn_kernel<H, D, STAGES>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         SpLayout<H, D, STAGES>::BYTES);
    configured = true;
  }
  const int rows = p.B * p.Lq;
  if (p.nsplit > 1 && cudaMemsetAsync(p.counters, 0, (size_t)rows * sizeof(int), stream) != cudaSuccess)
    return cudaErrorUnknown;
  LaunchScope ls("sparse_attn", stream);
  sparse_attn_kernel<H, D, STAGES><<<dim3(rows, p.nsplit), NT, SpLayout<H, D, STAGES>::BYTES, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_sparse(const SpParams& p, int H, int D, cudaStream_t stream) {
  const bool one_tile = p.split_slots <= 128;  // one tile per CTA: a single stage suffices
  if (H == 64 && D == 128) return one_tile ? launch_t<64, 128, 1>(p, stream) : launch_t<64, 128, 2>(p, stream);
  if (H == 16 && D == 64) return one_tile ? launch_t<16, 64, 1>(p, stream) : launch_t<16, 64, 2>(p, stream);
  return cudaErrorInvalidValue;
}

}  // namespace sparse
}  // namespace hs2
