// KV Bridging projection as one batched GEMM (tcgen05).
//
//   KV[l][kv] (T x d) = H (T x hidden) . W[l][kv] (hidden x d),  l < n_layers, kv in {K, V}
//
// All 2*n_layers products share the A operand H, so they are one GEMM against the
// concatenated [W[0][0] | W[0][1] | W[1][0] | ...] (hidden x 2*n_layers*d). Tiles: M = 128 rows of
// H (K-major A), N = 256 = two (layer, K/V) slices side by side (MN-major B read straight from
// W's row-major [hidden x d] slices, four 64-column blocks), K stepped 64 at a time through a
// 4-stage TMA ring. Accumulators live in TMEM, double-buffered (2 x 256 columns) so the epilogue
// of one tile overlaps the main loop of the next. Persistent CTAs walk the tiles M-major so the
// N-tiles of one H row block run back to back and re-hit L2.
//
// Warp roles (192 threads): warp 0 = TMA producer, warp 1 = MMA issuer + TMEM owner,
// warps 2..5 = epilogue (TMEM -> registers -> bf16 -> global).
#include "decode.h"
#include "host_util.h"
#include "prefill.h"
#include "tc.cuh"

namespace hs2 {
namespace bridge {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;       // 16 KB
constexpr int B_BYTES = BN * BK * 2;       // 32 KB (4 blocks of 64 columns x 64 k-rows)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NTHREADS = 192;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES;

struct Params {
  int T, hidden, n_slices, d;  // n_slices = 2 * n_layers
  int m_tiles, n_tiles;        // n_tiles = n_slices * d / BN
  __nv_bfloat16* out;          // [n_slices][T][d]
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

// B tile for output columns [n0, n0 + 256): slice s = n0 / d and the following ones; each 64-column
// block comes from W slice (col / d), columns (col % d) .. +63.
__global__ void __launch_bounds__(NTHREADS, 1)
    bridge_gemm_kernel(const __grid_constant__ CUtensorMap tmH, const __grid_constant__ CUtensorMap tmW, Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], acc_full[2], acc_empty[2];
  __shared__ uint32_t tmem_base;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x / 32, lane = threadIdx.x & 31;
  const int n_tiles_total = p.m_tiles * p.n_tiles;
  const int k_steps = p.hidden / BK;
  const long long limit = p.wait_ns;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], 1); }
    for (int i = 0; i < 2; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
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
      tma_prefetch_desc(&tmH);
      tma_prefetch_desc(&tmW);
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x) {
        const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % STAGES;
          if (!wait_abortable(&empty[s], ((it / STAGES) & 1) ^ 1, limit, &abort_flag, p.st, 501)) { ok = false; break; }
          uint8_t* sa = smem + s * STAGE_BYTES;
          uint8_t* sb = sa + A_BYTES;
          mbar_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(sa, &tmH, &full[s], ks * BK, mt * BM);
#pragma unroll
          for (int blk = 0; blk < BN / 64; ++blk) {
            const int col = nt * BN + blk * 64;
            const int slice = col / p.d, c0 = col % p.d;
            // W viewed as [n_slices * hidden rows x d]: rows slice*hidden + ks*BK .. +63
            tma_load_2d(sb + blk * (BK * 128), &tmW, &full[s], c0, slice * p.hidden + ks * BK);
          }
        }
      }
      if (!ok)
        for (uint32_t j = (it > STAGES ? it - STAGES : 0); j < it; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1, limit);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = idesc_bf16(BM, BN, 0, 1);
      uint32_t it = 0;
      int local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < n_tiles_total && ok; tile += gridDim.x, ++local) {
        const int ab = local & 1;
        if (!wait_abortable(&acc_empty[ab], ((local >> 1) & 1) ^ 1, limit, &abort_flag, p.st, 511)) { ok = false; break; }
        tc_fence_after();
        for (int ks = 0; ks < k_steps; ++ks, ++it) {
          const int s = it % STAGES;
          if (!wait_abortable(&full[s], (it / STAGES) & 1, limit, &abort_flag, p.st, 512)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + s * STAGE_BYTES), sb = sa + A_BYTES;
          const uint64_t da = sdesc(sa, 16, 1024), db = sdesc(sb, BK * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t a = sdesc_at(da, kk * 32);
            const uint64_t b = sdesc_at(db, kk * 2048);
            umma_ss(tmem + ab * BN, a, b, IDESC, (ks > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
    }
  } else {
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    int local = 0;
    for (int tile = blockIdx.x; tile < n_tiles_total; tile += gridDim.x, ++local) {
      const int ab = local & 1;
      int okw = __all_sync(0xffffffffu, mbar_try_wait(smem_u32(&acc_full[ab]), (local >> 1) & 1));
      if (!okw) {  // not complete yet: lane 0 waits (bounded) and passes the answer on
        if (lane == 0) okw = wait_abortable(&acc_full[ab], (local >> 1) & 1, limit, &abort_flag, p.st, 521) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
      }
      if (!okw) break;
      tc_fence_after();
      const int mt = tile / p.n_tiles, nt = tile % p.n_tiles;
      const int grow = mt * BM + row;
#pragma unroll 1
      for (int c = 0; c < BN; c += 32) {
        float v[32];
        tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + ab * BN + c, v);
        tmem_ld_wait();
        const int col = nt * BN + c;
        const int slice = col / p.d, c0 = col % p.d;
        if (grow < p.T) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) pk[x] = pack_bf16x2(v[2 * x], v[2 * x + 1]);
          uint4* dst = reinterpret_cast<uint4*>(p.out + ((size_t)slice * p.T + grow) * p.d + c0);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) { tc_fence_after(); tmem_dealloc(tmem, 512); }
}

}  // namespace bridge

namespace prefill {

hs2_status run_bridge(const hs2_bf16* Hs, int T, int hidden, const hs2_bf16* W, int n_layers, int d, hs2_bf16* KV,
                      DevStatus* st, cudaStream_t stream) {
  using namespace bridge;
  const int n_slices = 2 * n_layers;
  if ((n_slices * d) % BN != 0) return HS2_ERR_UNSUPPORTED_SHAPE;  // two 128-wide or four 64-wide slices per tile
  CUtensorMap tmH, tmW;
  if (!make_tmap_2d(&tmH, Hs, hidden, T, hidden, BK, BM)) return HS2_ERR_CUDA;
  if (!make_tmap_2d(&tmW, W, d, (uint64_t)n_slices * hidden, d, 64, BK)) return HS2_ERR_CUDA;
  Params p;
  p.T = T; p.hidden = hidden; p.n_slices = n_slices; p.d = d;
  p.m_tiles = (T + BM - 1) / BM;
  p.n_tiles = n_slices * d / BN;
  p.out = reinterpret_cast<__nv_bfloat16*>(KV);
  p.wait_ns = wait_limit_ns();
  p.st = st;
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(bridge_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    configured = true;
  }
  const int tiles = p.m_tiles * p.n_tiles;
  const int sms = num_sms();
  const int grid = tiles < sms ? tiles : sms;
  {
    LaunchScope ls("bridge_gemm", stream);
    bridge_gemm_kernel<<<grid, NTHREADS, SMEM_BYTES, stream>>>(tmH, tmW, p);
  }
  return cudaGetLastError() == cudaSuccess ? HS2_OK : HS2_ERR_CUDA;
}

}  // namespace prefill
}  // namespace hs2
