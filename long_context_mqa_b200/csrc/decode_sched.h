// Work schedule of the fused decode kernel, shared by the kernel, the selection kernels that read
// its partial records, and the host-side workspace sizing.
//
// Sequences are taken in groups of `gs` (the host picks gs from a K-bytes budget). For each group the
// flattened (sequence, 128-key tile) space is cut into G contiguous ranges, one per CTA; a range
// may cross a sequence boundary, so a CTA handles one or more "segments" per group. Sequence b
// is covered by CTAs c_lo(b)..c_hi(b) of its group, and CTA c's partial record for b sits at
// slot b * cmax + (c - c_lo(b)): the records of one sequence are contiguous.
//
// Index arithmetic is 32-bit inside a group (the host checks gtiles * G < 2^32).
#pragma once
#include <stdint.h>

namespace hs2 {
namespace dec {

struct Sched {
  int B, tps, G, gs, n_groups, cmax;

  __host__ __device__ long long gbase(int g) const { return (long long)g * gs * tps; }
  __host__ __device__ unsigned gtiles(int g) const {
    const int b1 = (g + 1) * gs < B ? (g + 1) * gs : B;
    return (unsigned)(b1 - g * gs) * (unsigned)tps;
  }
  // tiles [t0, t1) of CTA c in group g (flattened over all sequences)
  __host__ __device__ void range(int g, int c, long long& t0, long long& t1) const {
    const unsigned T = gtiles(g);
    t0 = gbase(g) + T * (unsigned)c / (unsigned)G;
    t1 = gbase(g) + T * (unsigned)(c + 1) / (unsigned)G;
  }
  // CTA of group g whose range holds flattened tile x
  __host__ __device__ int cta_of(int g, long long x) const {
    const unsigned T = gtiles(g);
    return (int)((((unsigned)(x - gbase(g)) + 1u) * (unsigned)G - 1u) / T);
  }
  // CTAs c_lo..c_hi of group g cover sequence b's tiles
  __host__ __device__ void covering(int b, int& g, int& c_lo, int& c_hi) const {
    g = b / gs;
    c_lo = cta_of(g, (long long)b * tps);
    c_hi = cta_of(g, (long long)(b + 1) * tps - 1);
  }
  __host__ __device__ int slot(int b, int c, int c_lo) const { return b * cmax + (c - c_lo); }
};

}  // namespace dec
}  // namespace hs2
