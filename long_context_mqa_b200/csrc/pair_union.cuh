// The union of the selections of two adjacent query rows of a sequence, for kernels that process
// the two rows together (their 64 heads each fill half of a 128-row MMA tile, and a key both rows
// selected is gathered, and its gradient added, once). Built by the whole (128-thread) block.
#pragma once
#include <stdint.h>

namespace hs2 {

constexpr int PAIR_MAX = 2 * 2048;  // union slots (two rows of up to 2,048 slots)

constexpr int UNION_NT = 128;  // the block

// Block-ordered compaction: appends, in index order, every i in [0, n) with keep(i) true to out
// via emit(position, i); returns the number kept. n <= 128 * 32.
template <class Keep, class Emit>
__device__ __forceinline__ int block_compact(int n, int base, Keep keep, Emit emit, int* s_warp) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int per = (n + UNION_NT - 1) / UNION_NT;
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
  for (int x = 0; x < UNION_NT / 32; ++x) {
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
// outside [0, Lk) are left out and set `bad`. `stage` holds 2 x `half` ints of shared memory for
// the two lists (S <= PAIR_MAX / 2); s_n holds 6 ints, s_warp 4. Every thread of the block calls
// it.
__device__ __forceinline__ int pair_union(const int32_t* idx, int S, int Lk, int r0, bool two, int32_t* stage,
                                          int32_t* ukey, uint8_t* uflag, int* s_warp, int* s_n, bool& bad) {
  const int tid = threadIdx.x;
  int32_t* A = stage;
  int32_t* Bl = stage + PAIR_MAX / 2;
  const int nBl = two ? S : 0;
  {
    // every load in flight before the first store (the lists come from global memory)
    constexpr int PER = (PAIR_MAX / 2 + UNION_NT - 1) / UNION_NT;
    int ra[PER], rb[PER];
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int i = tid + k * UNION_NT;
      ra[k] = i < S ? __ldg(idx + (size_t)r0 * S + i) : -1;
      rb[k] = i < nBl ? __ldg(idx + (size_t)(r0 + 1) * S + i) : -1;
    }
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int i = tid + k * UNION_NT;
      if (i < S) A[i] = ra[k];
      if (i < nBl) Bl[i] = rb[k];
    }
  }
  __syncthreads();
  auto sorted_tail = [&](const int32_t* L, int n) -> bool {
    bool good = true;
    for (int i = tid; i + 1 < n; i += UNION_NT) {
      const int a = L[i], nx = L[i + 1];
      good &= a == -1 ? nx == -1 : (nx == -1 || nx > a);
    }
    return good;
  };
  const bool merge = __syncthreads_and(sorted_tail(A, S) && sorted_tail(Bl, nBl)) != 0;
  auto in_range = [&](int j) { return j >= 0 && j < Lk; };
  {
    bool my_bad = false;
    for (int i = tid; i < S; i += UNION_NT) my_bad |= A[i] != -1 && !in_range(A[i]);
    for (int i = tid; i < nBl; i += UNION_NT) my_bad |= Bl[i] != -1 && !in_range(Bl[i]);
    if (my_bad) bad = true;
  }
  if (merge) {
    // A merge path over the two ascending lists. The in-range keys of each form a window of its
    // valid prefix (keys below 0 lead it, keys at or above Lk end it). Thread tid merges the
    // outputs [d0, d1) of the merged order (ties: A first), found by one co-rank search; a key
    // in both lists is written once, with both bits, by whoever takes it from A (the B cursor
    // then points at its copy, which is skipped when reached since A's previous key equals it).
    if (tid < 6) s_n[tid] = 0;
    __syncthreads();
    {
      int negA = 0, bigA = 0, negB = 0, bigB = 0;
      for (int i = tid; i < S; i += UNION_NT) {
        const int a = A[i];
        if (a != -1) {
          negA += a < 0;
          bigA += a >= Lk;
          if (i + 1 == S || A[i + 1] == -1) s_n[0] = i + 1;
        }
      }
      for (int i = tid; i < nBl; i += UNION_NT) {
        const int v = Bl[i];
        if (v != -1) {
          negB += v < 0;
          bigB += v >= Lk;
          if (i + 1 == nBl || Bl[i + 1] == -1) s_n[1] = i + 1;
        }
      }
      if (negA) atomicAdd(&s_n[2], negA);
      if (bigA) atomicAdd(&s_n[3], bigA);
      if (negB) atomicAdd(&s_n[4], negB);
      if (bigB) atomicAdd(&s_n[5], bigB);
    }
    __syncthreads();
    const int32_t* Ap = A + s_n[2];
    const int32_t* Bp = Bl + s_n[4];
    const int na = s_n[0] - s_n[3] - s_n[2], nb = s_n[1] - s_n[5] - s_n[4];
    const int total = na + nb;
    const int chunk = (total + UNION_NT - 1) / UNION_NT;
    const int d0 = tid * chunk < total ? tid * chunk : total;
    const int d1 = d0 + chunk < total ? d0 + chunk : total;
    int i0 = d0 - nb > 0 ? d0 - nb : 0;
    {
      int hi = d0 < na ? d0 : na;
      while (i0 < hi) {
        const int mid = (i0 + hi) >> 1;
        if (Ap[mid] <= Bp[d0 - mid - 1]) i0 = mid + 1; else hi = mid;
      }
    }
    const int j0 = d0 - i0;
    // pass 1 counts this thread's outputs, pass 2 writes them after a block scan
    int cnt = 0;
    {
      int i = i0, j = j0;
      for (int d = d0; d < d1; ++d) {
        if (j >= nb || (i < na && Ap[i] <= Bp[j])) { ++cnt; ++i; }
        else { cnt += !(i > 0 && Ap[i - 1] == Bp[j]); ++j; }
      }
    }
    const int lane = tid & 31, w = tid >> 5;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[w] = incl;
    __syncthreads();
    int pos = incl - cnt, U = 0;
#pragma unroll
    for (int x = 0; x < UNION_NT / 32; ++x) {
      pos += x < w ? s_warp[x] : 0;
      U += s_warp[x];
    }
    {
      int i = i0, j = j0;
      for (int d = d0; d < d1; ++d) {
        if (j >= nb || (i < na && Ap[i] <= Bp[j])) {
          ukey[pos] = Ap[i];
          uflag[pos] = (uint8_t)(1u | (j < nb && Bp[j] == Ap[i] ? 2u : 0u));
          ++pos;
          ++i;
        } else {
          if (!(i > 0 && Ap[i - 1] == Bp[j])) {
            ukey[pos] = Bp[j];
            uflag[pos] = 2u;
            ++pos;
          }
          ++j;
        }
      }
    }
    __syncthreads();  // s_warp and the lists are reused
    return U;
  }
  const int u0 = block_compact(S, 0, [&](int i) { return in_range(A[i]); },
                               [&](int pos, int i) { ukey[pos] = A[i]; uflag[pos] = 1u; }, s_warp);
  const int u1 = block_compact(nBl, u0, [&](int i) { return in_range(Bl[i]); },
                               [&](int pos, int i) { ukey[pos] = Bl[i]; uflag[pos] = 2u; }, s_warp);
  return u0 + u1;
}

}  // namespace hs2
