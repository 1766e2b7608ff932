// stem_select_row.cuh — selection of one CSR row's key blocks by one warp.
//
// AngelSlim documentation §2.2 (sink and window blocks always kept), "Stem"
// gist.science zh §2.1 (the position-decay budget b of the row), youleyou
// HPC-BSA article §3.1 (the compacted, ascending list the attention walks):
// keep the forced blocks F, then the m = min(max(b - |F|, 0), c - |F|) best
// other causal blocks by (score descending, index ascending), NaN ranked as
// -inf; write them in ascending order.  One warp per row: the scoring kernel
// selects the rows it has just scored with it, and select_kernel runs it on
// given scores.
#pragma once

#include "stem_device.cuh"
#include "stem_internal.h"

namespace stem {

// Order-preserving 32-bit key of a float (larger float, larger key); NaN ranks
// as -inf, and -0 and +0 get the same key (they compare equal as numbers, so
// the lower block index wins between them, as for any other tie).
__device__ __forceinline__ uint32_t order_key(float f) {
  if (f != f) f = -__int_as_float(0x7f800000);
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ int warp_exclusive_scan(int x) {
  const int lane = lane_id();
  int incl = x;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  return incl - x;
}

// row: the row's block scores (index = key block, local to the sequence), at
// least i + 1 of them; with group > 1 the rows of the group's other query
// heads follow at multiples of head_stride, and a block's key is the best of
// the group's scores (order_key is monotone and maps NaN below every number).
// keys: this warp's scratch (>= i + 1 entries); hist: this warp's scratch of
// 256 ints; the list (b entries, ascending) is written to
// col_idx + row_ptr[r + e row_stride] for each of the group's heads e.
static __device__ __noinline__ void warp_select_row_group(const float* __restrict__ row, size_t head_stride,
                                                          int group, int i, int b, int sink, int window,
                                                          uint32_t* keys, int* hist, int32_t* __restrict__ col_idx,
                                                          const int32_t* __restrict__ row_ptr, size_t r,
                                                          size_t row_stride) {
  const int lane = lane_id();
  const int c = i + 1;
  const int nforced = static_cast<int>(forced_count(i, sink, window));
  const int ncand = c - nforced;
  const int m = min(max(b - nforced, 0), ncand);  // candidates to pick
  const bool all = (m == ncand);
  uint32_t thr = 0u;
  int take_eq = 0;  // candidates equal to thr to take, lowest index first
  if (m > 0 && !all) {
    for (int j = lane; j < c; j += 32) {
      uint32_t k = order_key(row[j]);
      for (int e = 1; e < group; ++e) k = max(k, order_key(row[e * head_stride + j]));
      keys[j] = k;
    }
    __syncwarp();
    // radix select of the m-th largest candidate key, 8 bits per pass
    uint32_t prefix = 0u;
    int need = m;
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int q = lane; q < 256; q += 32) hist[q] = 0;
      __syncwarp();
      const uint32_t hmask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
      for (int j = lane; j < c; j += 32) {
        if (is_forced(j, i, sink, window)) continue;
        const uint32_t k = keys[j];
        if ((k & hmask) == prefix) atomicAdd(&hist[(k >> shift) & 0xFFu], 1);
      }
      __syncwarp();
      // lane L holds digits 255 - 8L .. 248 - 8L, highest first
      int mine[8];
      int tot = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        mine[q] = hist[255 - 8 * lane - q];
        tot += mine[q];
      }
      const int before = warp_exclusive_scan(tot);
      const unsigned hit = __ballot_sync(0xffffffffu, before + tot >= need);
      const int src = __ffs(hit) - 1;  // the count of this prefix class is >= need
      int digit = 0, acc = 0;
      if (lane == src) {
        acc = before;
        int q = 0;
        for (; q < 7; ++q) {
          if (acc + mine[q] >= need) break;
          acc += mine[q];
        }
        digit = 255 - 8 * lane - q;
      }
      digit = __shfl_sync(0xffffffffu, digit, src);
      acc = __shfl_sync(0xffffffffu, acc, src);
      need -= acc;
      prefix |= static_cast<uint32_t>(digit) << shift;
      __syncwarp();  // the histogram is cleared again by the next pass
    }
    thr = prefix;
    take_eq = need;
  }
  // Emit forced blocks, candidates above the threshold and the first take_eq
  // equal to it, ascending: each lane owns a contiguous run of indices.
  const int per = (c + 31) / 32;
  const int j0 = min(c, lane * per);
  const int j1 = min(c, j0 + per);
  int n_eq = 0;
  if (m > 0 && !all)
    for (int j = j0; j < j1; ++j)
      if (!is_forced(j, i, sink, window) && keys[j] == thr) ++n_eq;
  const int eq_before = warp_exclusive_scan(n_eq);
  auto take = [&](int j, int& e) -> bool {
    if (is_forced(j, i, sink, window)) return true;
    if (m <= 0) return false;
    if (all) return true;
    const uint32_t k = keys[j];
    const bool sel = k > thr || (k == thr && e < take_eq);
    if (k == thr) ++e;
    return sel;
  };
  int n_sel = 0;
  {
    int e = eq_before;
    for (int j = j0; j < j1; ++j) n_sel += take(j, e);
  }
  const int pos0 = warp_exclusive_scan(n_sel);
  for (int h = 0; h < group; ++h) {
    int32_t* __restrict__ out = col_idx + row_ptr[r + h * row_stride];
    int e = eq_before, pos = pos0;
    for (int j = j0; j < j1; ++j)
      if (take(j, e)) out[pos++] = j;
  }
  __syncwarp();
}

// One query head's row (the fused selection of the scoring kernel).
static __device__ __forceinline__ void warp_select_row(const float* __restrict__ row, int i, int b, int sink,
                                                       int window, uint32_t* keys, int* hist,
                                                       int32_t* __restrict__ col_idx,
                                                       const int32_t* __restrict__ row_ptr, size_t r) {
  warp_select_row_group(row, 0, 1, i, b, sink, window, keys, hist, col_idx, row_ptr, r, 0);
}

}  // namespace stem
