// Work schedule of the fused decode kernel, shared by the kernel, the selection kernels that read
// its partial records, and the host-side workspace sizing.
//
// Sequences are taken in groups of `gs` (the host uses one group of all sequences). The flattened
// (sequence, 128-key tile) space of a group is cut into G contiguous ranges, one per CTA, by a
// table of start tiles; a range may cross a sequence boundary, so a CTA handles one or more
// "segments" per group. Sequence b
// is covered by CTAs c_lo(b)..c_hi(b) of its group, and CTA c's partial record for b sits at
// slot b * cmax + (c - c_lo(b)): the records of one sequence are contiguous.
//
// Index arithmetic is 32-bit inside a group.
#pragma once
#include <stdint.h>

namespace hs2 {
namespace dec {

constexpr int kMaxCtas = 256;

struct Sched {
  int B, tps, G, gs, n_groups, cmax;
  // CTA c covers flattened tiles [start[c], start[c + 1]) of each group (the host uses one group)
  unsigned start[kMaxCtas + 1];

  __host__ __device__ long long gbase(int g) const { return (long long)g * gs * tps; }
  __host__ __device__ unsigned gtiles(int g) const {
    const int b1 = (g + 1) * gs < B ? (g + 1) * gs : B;
    return (unsigned)(b1 - g * gs) * (unsigned)tps;
  }
  // tiles [t0, t1) of CTA c in group g (flattened over all sequences)
  __host__ __device__ void range(int g, int c, long long& t0, long long& t1) const {
    t0 = gbase(g) + start[c];
    t1 = gbase(g) + start[c + 1];
  }
  // CTA of group g whose range holds flattened tile x (the last CTA starting at or before it)
  __host__ __device__ int cta_of(int g, long long x) const {
    const unsigned y = (unsigned)(x - gbase(g));
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (start[mid] <= y) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  // CTAs c_lo..c_hi of group g cover sequence b's tiles
  __host__ __device__ void covering(int b, int& g, int& c_lo, int& c_hi) const {
    g = b / gs;
    c_lo = cta_of(g, (long long)b * tps);
    c_hi = cta_of(g, (long long)(b + 1) * tps - 1);
  }
  __host__ __device__ int slot(int b, int c, int c_lo) const { return b * cmax + (c - c_lo); }

  // Host: cut the T = gs * tps tiles of a group into G ranges. A CTA whose range crosses a
  // sequence boundary runs two segments, which cost about `beta` tiles more (a pipeline drain,
  // an output record, the next sequence's logsumexp), so it takes beta fewer tiles; everything
  // else is split evenly. Used when each range is far shorter than a sequence (so it crosses
  // at most one boundary); otherwise an even split. Every CTA gets at least one tile (G <= T).
  void partition(int beta) {
    const unsigned T = gtiles(0);
    const bool adjust = beta > 0 && gs > 1 && T / (unsigned)G >= 4u * (unsigned)beta &&
                        (unsigned)tps >= 2u * (T / (unsigned)G);
    long long units_left = (long long)T + (adjust ? (long long)beta * (gs - 1) : 0);
    unsigned pos = 0;
    start[0] = 0;
    for (int c = 0; c < G; ++c) {
      unsigned end;
      if (c == G - 1) {
        end = T;
      } else {
        const long long u = (units_left + (G - c) / 2) / (G - c);
        end = pos + (unsigned)(u > 1 ? u : 1);
        bool crossed = false;
        if (adjust) {
          const unsigned seq_end = (pos / (unsigned)tps + 1) * (unsigned)tps;
          if (end > seq_end) {
            if (end - (unsigned)beta > seq_end) { end -= (unsigned)beta; crossed = true; }
            else end = seq_end;
          }
        }
        const unsigned max_end = T - (unsigned)(G - 1 - c);  // one tile left for each later CTA
        if (end > max_end) end = max_end;
        if (end <= pos) end = pos + 1;
        units_left -= (long long)(end - pos) + (crossed ? beta : 0);
      }
      start[c + 1] = end;
      pos = end;
    }
  }
};

}  // namespace dec
}  // namespace hs2
