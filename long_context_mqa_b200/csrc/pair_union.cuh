// The union of the selections of two adjacent query rows of a sequence, for kernels that process
// the two rows together (their 64 heads each fill half of a 128-row MMA tile, and a key both rows
// selected is gathered, and its gradient added, once). 128 threads.
#pragma once
#include <stdint.h>

namespace hs2 {

constexpr int PAIR_MAX = 2 * 2048;  // union slots (two rows of up to 2,048 slots)

// Block-ordered compaction (128 threads): appends, in index order, every i in [0, n) with
// keep(i) true to out via emit(position, i); returns the number kept. n <= 128 * 32.
template <class Keep, class Emit>
__device__ __forceinline__ int block_compact(int n, int base, Keep keep, Emit emit, int* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int per = (n + 127) / 128;
  const int i0 = tid * per;
  unsigned mine = 0;  // bit x: element i0 + x kept (per <= 32)
  for (int x = 0; x < per; ++x)
    if (i0 + x < n && keep(i0 + x)) mine |= 1u << x;
  const int cnt = __popc(mine);
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) s_warp[w] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int x = 0; x < 4; ++x) {
    before += x < w ? s_warp[x] : 0;
    total += s_warp[x];
  }
  int pos = base + before + incl - cnt;
  for (int x = 0; x < per; ++x)
    if ((mine >> x) & 1u) emit(pos++, i0 + x);
  __syncthreads();  // s_warp is reused by the next call
  return total;
}

// Builds the union of rows r0 and r0 + 1 (the second only if `two`) of idx [rows][S] into ukey /
// uflag (bit 0: row r0 selected the key, bit 1: row r0 + 1) and returns its size. Lists that are
// strictly ascending with any -1 slots at the tail (the full layer's output) are merged without
// duplicates; any other lists are concatenated, each slot once (as the forward counts them). Keys
// outside [0, Lk) are left out and set `bad`. `stage` holds 2 x 2,048 ints of shared memory for
// the two lists (binary searches run there). Every thread of the block calls it.
__device__ __forceinline__ int pair_union(const int32_t* idx, int S, int Lk, int r0, bool two, int32_t* stage,
                                          int32_t* ukey, uint8_t* uflag, int* s_warp, int* s_n, bool& bad) {
  const int tid = threadIdx.x;
  int32_t* A = stage;
  int32_t* Bl = stage + PAIR_MAX / 2;
  const int nBl = two ? S : 0;
  for (int i = tid; i < S; i += 128) A[i] = __ldg(idx + (size_t)r0 * S + i);
  for (int i = tid; i < nBl; i += 128) Bl[i] = __ldg(idx + (size_t)(r0 + 1) * S + i);
  __syncthreads();
  auto sorted_tail = [&](const int32_t* L, int n) -> bool {
    bool good = true;
    for (int i = tid; i + 1 < n; i += 128) {
      const int a = L[i], nx = L[i + 1];
      good &= a == -1 ? nx == -1 : (nx == -1 || nx > a);
    }
    return good;
  };
  const bool merge = __syncthreads_and(sorted_tail(A, S) && sorted_tail(Bl, nBl));
  auto in_range = [&](int j) { return j >= 0 && j < Lk; };
  {
    bool my_bad = false;
    for (int i = tid; i < S; i += 128) my_bad |= A[i] != -1 && !in_range(A[i]);
    for (int i = tid; i < nBl; i += 128) my_bad |= Bl[i] != -1 && !in_range(Bl[i]);
    if (my_bad) bad = true;
  }
  if (merge) {
    // the valid prefix of each list
    if (tid == 0) { s_n[0] = 0; s_n[1] = 0; }
    __syncthreads();
    for (int i = tid; i < S; i += 128)
      if (A[i] != -1 && (i + 1 == S || A[i + 1] == -1)) s_n[0] = i + 1;
    for (int i = tid; i < nBl; i += 128)
      if (Bl[i] != -1 && (i + 1 == nBl || Bl[i + 1] == -1)) s_n[1] = i + 1;
    __syncthreads();
    const int nA = s_n[0], nB = s_n[1];
    auto find = [&](const int32_t* L, int n, int key) -> bool {  // binary search, L ascending
      int lo = 0, hi = n - 1;
      while (lo <= hi) {
        const int mid = (lo + hi) >> 1, v = L[mid];
        if (v == key) return true;
        if (v < key) lo = mid + 1; else hi = mid - 1;
      }
      return false;
    };
    const int u0 = block_compact(nA, 0, [&](int i) { return in_range(A[i]); },
                                 [&](int pos, int i) {
                                   ukey[pos] = A[i];
                                   uflag[pos] = (uint8_t)(1u | (find(Bl, nB, A[i]) ? 2u : 0u));
                                 }, s_warp);
    const int u1 = block_compact(nB, u0, [&](int i) { return in_range(Bl[i]) && !find(A, nA, Bl[i]); },
                                 [&](int pos, int i) { ukey[pos] = Bl[i]; uflag[pos] = 2u; }, s_warp);
    return u0 + u1;
  }
  const int u0 = block_compact(S, 0, [&](int i) { return in_range(A[i]); },
                               [&](int pos, int i) { ukey[pos] = A[i]; uflag[pos] = 1u; }, s_warp);
  const int u1 = block_compact(nBl, u0, [&](int i) { return in_range(Bl[i]); },
                               [&](int pos, int i) { ukey[pos] = Bl[i]; uflag[pos] = 2u; }, s_warp);
  return u0 + u1;
}

}  // namespace hs2
