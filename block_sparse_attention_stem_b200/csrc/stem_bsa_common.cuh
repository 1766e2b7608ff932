// stem_bsa_common.cuh — pieces shared by the two block-sparse attention kernels
// (one CSR row per CTA, and a pair of query heads with one shared list per
// CTA): tile geometry, block-list staging and walking, and the exp2 chunk.
#pragma once

#include "stem_device.cuh"
#include "stem_kernels.h"

namespace stem {
namespace {

constexpr int kHalf = 64;               // keys per S buffer
constexpr int kMaxList = 2048;          // list entries per tile staged in SMEM
// Pairs of keys (bit k: keys 2k, 2k+1 of a 32-key chunk) whose exp2 runs on
// the FMA pipes (exp2_poly2) instead of the MUFU unit, off the diagonal block.
#ifndef STEM_BSA_POLY_MASK
#define STEM_BSA_POLY_MASK 0x0u
#endif
constexpr uint32_t kPolyMask = STEM_BSA_POLY_MASK;

template <bool kFp8>
struct BsaCfg {
  static constexpr int kQBytes = kFp8 ? 16384 : 32768;     // one 128 x 128 Q block
  static constexpr int kKHalfBytes = kFp8 ? 8192 : 16384;  // 64 keys x 128 dims of K
  static constexpr int kVHalfBytes = 16384;                // 64 keys x 128 dims of V (bf16 or f16)
  static constexpr int kKSlabs = kFp8 ? 1 : 2;             // 128-byte head-dim slabs per K row
  static constexpr float kRescaleLog2 = 8.f;               // max growth before O is rescaled
};
template struct BsaCfg<true>;

struct Tile {
  bool valid;    // the CTA's second tile may not exist
  int i, h, hk;  // query block, query head, KV head
  int beg, end;  // CSR range
};

// Next valid list entry at or after position p: 0 <= j <= i and strictly
// above the previous valid entry.  Returns the entry's position or `end`.
__device__ __forceinline__ int next_valid(const int32_t* __restrict__ col, int p, int end, int prev, int i,
                                          int* j_out) {
  for (; p < end; ++p) {
    const int j = __ldg(col + p);
    if (j >= 0 && j <= i && j > prev) {
      *j_out = j;
      return p;
    }
  }
  return end;
}

// Walks the valid entries of a tile's list in order: from SMEM when staged,
// otherwise straight from global memory.
struct ListCursor {
  int p, prev;
  __device__ __forceinline__ explicit ListCursor(int beg) : p(beg), prev(-1) {}
  __device__ __forceinline__ int next(const int32_t* smem_list, bool in_smem, int n, const int32_t* col, int end,
                                      int i) {
    if (in_smem) return smem_list[n];
    int j = 0;
    p = next_valid(col, p, end, prev, i, &j) + 1;
    prev = j;
    return j;
  }
};

// Stage the valid entries of one list into SMEM (one whole warp).  Well-formed
// lists (every entry in [0, i], strictly ascending) are copied 32 at a time; a
// malformed list is compacted entry by entry and reported.
__device__ void stage_list(const int32_t* __restrict__ col, const Tile& t, int32_t* dst, int* nvalid,
                           int* in_smem, int* status) {
  const int lane = lane_id();
  if (!t.valid) {
    if (lane == 0) { *nvalid = 0; *in_smem = 1; }
    return;
  }
  bool good = true;
  for (int p0 = t.beg; p0 < t.end; p0 += 32) {
    const int p = p0 + lane;
    const int j = p < t.end ? __ldg(col + p) : 0;
    int before = __shfl_up_sync(0xffffffffu, j, 1);
    if (lane == 0) before = p0 > t.beg ? __ldg(col + p0 - 1) : -1;
    const bool bad = p < t.end && (j < 0 || j > t.i || j <= before);
    if (__any_sync(0xffffffffu, bad)) { good = false; break; }
    if (p < t.end && p - t.beg < kMaxList) dst[p - t.beg] = j;
  }
  if (good) {
    if (lane == 0) { *nvalid = t.end - t.beg; *in_smem = (t.end - t.beg) <= kMaxList; }
    return;
  }
  if (lane == 0) {
    set_status(status, STEM_ERR_BAD_BLOCKLIST_CODE);
    int n = 0, prev = -1, j = 0;
    for (int p = next_valid(col, t.beg, t.end, prev, t.i, &j); p < t.end;
         p = next_valid(col, p + 1, t.end, prev, t.i, &j)) {
      if (n < kMaxList) dst[n] = j;
      prev = j;
      ++n;
    }
    *nvalid = n;
    *in_smem = n <= kMaxList;
  }
}

// p = exp2(s c - m) for one 32-key chunk of a row: packed scale-and-shift,
// exp2 (MUFU, or for the pairs in kPoly the FMA-pipe polynomial), packed row
// sums and bf16 (or f16) packing.  w[k] holds keys 2k (low half) and 2k + 1.
template <uint32_t kPoly, bool kF16>
__device__ __forceinline__ void exp_chunk(const uint32_t* rr, float2 c2, float2 nm2, float2& ps0, float2& ps1,
                                          uint32_t* w) {
#pragma unroll
  for (int x = 0; x < 16; x += 2) {
    const float2 a = ffma2(make_float2(__uint_as_float(rr[2 * x]), __uint_as_float(rr[2 * x + 1])), c2, nm2);
    const float2 a2 = ffma2(make_float2(__uint_as_float(rr[2 * x + 2]), __uint_as_float(rr[2 * x + 3])), c2, nm2);
    const float2 p01 = ((kPoly >> x) & 1u) ? exp2_poly2(a) : make_float2(fast_exp2(a.x), fast_exp2(a.y));
    const float2 p23 = ((kPoly >> (x + 1)) & 1u) ? exp2_poly2(a2) : make_float2(fast_exp2(a2.x), fast_exp2(a2.y));
    ps0 = fadd2(ps0, p01);
    ps1 = fadd2(ps1, p23);
    w[x] = kF16 ? f32x2_to_f16x2(p01.x, p01.y) : pack_bf16x2(p01.x, p01.y);
    w[x + 1] = kF16 ? f32x2_to_f16x2(p23.x, p23.y) : pack_bf16x2(p23.x, p23.y);
  }
}

}  // namespace
}  // namespace stem
