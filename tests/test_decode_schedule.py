"""Host logic of the decode work schedule (csrc/decode_sched.h), compiled for the CPU.

The fused decode kernel cuts the flattened (sequence, 128-key tile) space into one contiguous
range per CTA; the selection kernels find a sequence's CTAs and records through the same header.
These checks run the header's host code with g++ on ragged and uniform batches: every tile is
owned by exactly one CTA, every CTA has work, the lookups invert the tables, a CTA that crosses a
sequence boundary gives up the boundary's tiles, and the records of a sequence are contiguous.
"""
import json
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_SRC = r"""
#include <cstdio>
#include <cstdlib>
#include <vector>
#include "decode_sched.h"
using namespace hs2::dec;
int main(int argc, char** argv) {
  // argv: beta G len0 len1 ...
  const int beta = atoi(argv[1]), sms = atoi(argv[2]);
  std::vector<int> lens;
  for (int i = 3; i < argc; ++i) lens.push_back(atoi(argv[i]));
  static Sched s;
  s.set_lengths((int)lens.size(), lens.data());
  const long long T = s.tiles();
  s.G = (int)(T < sms ? T : sms);
  s.partition(beta);
  int cmax = 1;
  printf("{\"T\": %lld, \"G\": %d, \"start\": [", T, s.G);
  for (int c = 0; c <= s.G; ++c) printf("%s%u", c ? ", " : "", s.start[c]);
  printf("], \"seq_start\": [");
  for (int b = 0; b <= s.B; ++b) printf("%s%u", b ? ", " : "", s.seq_start[b]);
  printf("], \"cover\": [");
  for (int b = 0; b < s.B; ++b) {
    int g, lo, hi;
    s.covering(b, g, lo, hi);
    if (hi - lo + 1 > cmax) cmax = hi - lo + 1;
    printf("%s[%d, %d]", b ? ", " : "", lo, hi);
  }
  s.cmax = cmax;
  // seq_of and cta_of on every tile
  int bad = 0;
  for (long long t = 0; t < T; ++t) {
    const int b = s.seq_of(t), c = s.cta_of(0, t);
    if (!(s.seq_start[b] <= t && t < s.seq_start[b + 1])) ++bad;
    if (!(s.start[c] <= t && t < s.start[c + 1])) ++bad;
  }
  // slots of one sequence are consecutive and inside [b * cmax, (b + 1) * cmax)
  for (int b = 0; b < s.B; ++b) {
    int g, lo, hi;
    s.covering(b, g, lo, hi);
    for (int c = lo; c <= hi; ++c)
      if (s.slot(b, c, lo) != b * cmax + (c - lo) || c - lo >= cmax) ++bad;
  }
  printf("], \"cmax\": %d, \"lookup_errors\": %d}\n", cmax, bad);
  return 0;
}
"""


@pytest.fixture(scope="module")
def sched_bin(tmp_path_factory):
    gxx = shutil.which("g++")
    if gxx is None:
        pytest.skip("g++ not available")
    d = tmp_path_factory.mktemp("sched")
    src = d / "sched.cpp"
    src.write_text(_SRC)
    exe = d / "sched"
    subprocess.check_call([gxx, "-std=c++17", "-O1", "-D__host__=", "-D__device__=", "-D__forceinline__=inline",
                           "-I", os.path.join(ROOT, "long_context_mqa_b200", "csrc"), str(src), "-o", str(exe)])
    return str(exe)


def _run(exe, lens, sms=148, beta=4):
    out = subprocess.run([exe, str(beta), str(sms)] + [str(x) for x in lens], capture_output=True, text=True,
                         check=True).stdout
    return json.loads(out)


CASES = [
    [262144] * 8,                                   # the bench batch
    [1048576] * 2,
    [32768] * 32,
    [262144, 196608, 131072, 98304, 65536, 32768, 16384, 4096],  # the ragged clause
    [1, 128, 129, 40000, 777, 12345],
    [100, 1000, 1152, 1153, 3000],
    [5],
]


@pytest.mark.parametrize("lens", CASES)
def test_partition_covers_every_tile_once(sched_bin, lens):
    r = _run(sched_bin, lens)
    T, G, start = r["T"], r["G"], r["start"]
    assert T == sum((n + 127) // 128 for n in lens)
    assert G == min(T, 148)
    assert start[0] == 0 and start[-1] == T
    assert all(start[c + 1] > start[c] for c in range(G))     # every CTA has at least one tile
    assert r["lookup_errors"] == 0
    seq_start = r["seq_start"]
    for b, n in enumerate(lens):
        assert seq_start[b + 1] - seq_start[b] == (n + 127) // 128
        lo, hi = r["cover"][b]
        # the covering CTAs are exactly those whose ranges meet the sequence's tiles
        meets = [c for c in range(G) if start[c] < seq_start[b + 1] and start[c + 1] > seq_start[b]]
        assert meets == list(range(lo, hi + 1))
        assert hi - lo + 1 <= r["cmax"]


@pytest.mark.parametrize("lens", [[262144] * 8, [1048576] * 2])
def test_crossing_ranges_give_up_beta_tiles(sched_bin, lens):
    """With long sequences, a range that crosses a sequence boundary (two segments) holds about
    beta fewer tiles than the others, and the ranges are otherwise even."""
    beta = 4
    r = _run(sched_bin, lens, beta=beta)
    start, seq_start, G = r["start"], r["seq_start"], r["G"]
    crossing, plain = [], []
    for c in range(G):
        a, e = start[c], start[c + 1]
        crosses = any(a < s < e for s in seq_start[1:-1])
        (crossing if crosses else plain).append(e - a)
    assert plain and max(plain) - min(plain) <= 2
    if crossing:
        assert max(crossing) <= min(plain) - beta + 2
    r0 = _run(sched_bin, lens, beta=0)                      # beta 0: the even split
    sizes = [r0["start"][c + 1] - r0["start"][c] for c in range(r0["G"])]
    assert max(sizes) - min(sizes) <= 1
