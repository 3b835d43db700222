// The decode output of one (sequence, head), shared by the token-level and the block-level
// selection launches: the decode kernel's CTAs c_lo..c_hi covering sequence b left one
// unnormalised output record each (sums of p' v with p' = exp2(s c - lse2'), in consecutive
// slots from b * cmax); the output is their sum divided by L'_h = sum_j p'_jh (times an e4m3 V
// cache's scale). One warp, lane = 4 of the 128 columns.
#pragma once
#include "decode.h"
#include "tc.cuh"

namespace hs2 {

__device__ __forceinline__ void combine_decode_output(const float* opart, const float* lsum, float oscale,
                                                      __nv_bfloat16* out, int H, int D, const dec::Sched& sch,
                                                      DevStatus* st, int b, int h, unsigned lane) {
  int g, c_lo, c_hi;
  sch.covering(b, g, c_lo, c_hi);
  const int n_slots = c_hi - c_lo + 1;
  if (n_slots > sch.cmax || D != 128) {
    if (lane == 0) report_status(st, kStatusBounds, 303);
    return;
  }
  const float4* rec = reinterpret_cast<const float4*>(opart + ((size_t)sch.slot(b, c_lo, c_lo) * H + h) * D) + lane;
  const size_t rstride = (size_t)H * D / 4;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
  for (int i = 0; i < n_slots; ++i) {
    const float4 v = __ldcg(rec + i * rstride);
    acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
  }
  const float inv = oscale / lsum[b * H + h];  // the records are sums of p' v, p' unnormalised
  __nv_bfloat16* o = out + ((size_t)b * H + h) * D + 4 * lane;
  reinterpret_cast<__nv_bfloat162*>(o)[0] = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  reinterpret_cast<__nv_bfloat162*>(o)[1] = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
}

}  // namespace hs2
