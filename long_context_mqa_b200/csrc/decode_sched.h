// Work schedule of the fused decode kernel, shared by the kernel, the selection kernels that read
// its partial records, and the host-side workspace sizing.
//
// Sequence b (seq_len[b] tokens, any length: ragged batches are native) owns the 128-key tiles
// [seq_start[b], seq_start[b + 1]) of one flattened tile space, which a table of start tiles
// cuts into G contiguous ranges, one per CTA; a range may cross a sequence boundary, so a CTA
// handles one or more "segments". Sequence b is covered by CTAs c_lo(b)..c_hi(b), and CTA c's
// partial record for b sits at slot b * cmax + (c - c_lo(b)): the records of one sequence are
// contiguous. Index arithmetic is 32-bit (the host checks the tile count).
#pragma once
#include <stdint.h>

namespace hs2 {
namespace dec {

constexpr int kMaxCtas = 256;
constexpr int kMaxSeqs = 256;

struct Sched {
  int B, G, n_groups, cmax;          // n_groups is 1: one flattened range of all sequences' tiles
  unsigned start[kMaxCtas + 1];      // CTA c covers flattened tiles [start[c], start[c + 1])
  unsigned seq_start[kMaxSeqs + 1];  // sequence b's tiles are [seq_start[b], seq_start[b + 1])
  int seq_len[kMaxSeqs];             // sequence b's tokens (its last tile may be partial)

  __host__ __device__ unsigned tiles() const { return seq_start[B]; }
  // tiles [t0, t1) of CTA c (flattened over all sequences; g is 0)
  __host__ __device__ void range(int g, int c, long long& t0, long long& t1) const {
    (void)g;
    t0 = start[c];
    t1 = start[c + 1];
  }
  // the sequence holding flattened tile t
  __host__ __device__ int seq_of(long long t) const {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((long long)seq_start[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  // CTA whose range holds flattened tile x (the last CTA starting at or before it; g is 0)
  __host__ __device__ int cta_of(int g, long long x) const {
    (void)g;
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if ((long long)start[mid] <= x) lo = mid; else hi = mid - 1;
    }
    return lo;
  }
  // CTAs c_lo..c_hi cover sequence b's tiles
  __host__ __device__ void covering(int b, int& g, int& c_lo, int& c_hi) const {
    g = 0;
    c_lo = cta_of(0, seq_start[b]);
    c_hi = cta_of(0, (long long)seq_start[b + 1] - 1);
  }
  __host__ __device__ int slot(int b, int c, int c_lo) const { return b * cmax + (c - c_lo); }

  // Host: sequence lengths (each at least 1 token) -> the flattened tile space.
  void set_lengths(int nseq, const int* lens) {
    B = nseq;
    n_groups = 1;
    seq_start[0] = 0;
    for (int b = 0; b < nseq; ++b) {
      seq_len[b] = lens[b];
      seq_start[b + 1] = seq_start[b] + (unsigned)((lens[b] + 127) / 128);
    }
  }
  // Host: cut the tiles into G ranges (G <= tiles). A CTA whose range crosses a sequence boundary
  // runs two segments, which cost about `beta` tiles more (a pipeline drain, an output record,
  // the next sequence's logsumexp), so it takes beta fewer tiles; everything else is split
  // evenly. Every CTA gets at least one tile.
  void partition(int beta) {
    const unsigned T = tiles();
    const bool adjust = beta > 0 && B > 1 && T / (unsigned)G >= 4u * (unsigned)beta;
    long long units_left = (long long)T + (adjust ? (long long)beta * (B - 1) : 0);
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
          const unsigned seq_end = seq_start[seq_of(pos) + 1];
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
