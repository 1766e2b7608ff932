// k_bsa.cu — causal block-sparse flash attention over pre-compacted block lists.
//
// "Stem" gist.science zh §2.3 (exact softmax and aggregation only over the
// selected blocks); youleyou HPC-BSA article §3.1 (the inner loop walks a list
// prepared outside it; a skipped block is the same as a block of -inf scores,
// so the softmax needs no change; fixed 128 x 128 tiles).
//
// One CTA owns one CSR row: a 128-token query block of one query head.  For
// every listed key block j (ascending, the diagonal last):
//   S_n = Q K_j^T          tcgen05.mma, Q read from TMEM, K from SMEM, fp32 in
//                          TMEM (two S buffers)
//   P_n = exp2(S c - m)    softmax warps; P written back over the S buffer and
//                          read by the next MMA straight from TMEM
//   O  += P_n V_j          tcgen05.mma, V from SMEM (MN-major), fp32
//                          accumulator resident in TMEM
// The reference row max m moves (and O is rescaled in TMEM) only when a block
// raises it by more than a threshold (2^8 for bf16, 2^1 for fp8), so P stays
// bounded and rescales are rare; O and the row sums share that reference, so
// the result is exact.  Causal masking happens only on the diagonal block.
// The tensor core reads only K and V from shared memory.
//
// fp8: P would carry only three mantissa bits as one e4m3 value (up to 6%
// error per weight, which rows with few keys cannot average out), so it is
// split as P*224 = hi + lo with hi = e4m3(P*224) and lo = e4m3 of the
// remainder; two e4m3 MMAs accumulate hi.V and lo.V into the same O, which
// leaves P with about eight significant bits.
//
// Warp roles (320 threads):
//   warps 0-3  softmax, key columns 0-63 and O columns 0-63 (TMEM lane quarters 0-3)
//   warps 4-7  softmax, key columns 64-127 and O columns 64-127
//   warp  8    TMA producer: K_j, V_j of every listed block into a slot ring
//   warp  9    TMEM owner and single-thread MMA issuer
// The two softmax warpgroups exchange their partial row maxima through shared
// memory once per block (an mbarrier per block parity, so every wait is bounded).
#include "stem_device.cuh"
#include "stem_kernels.h"

namespace stem {

namespace {

constexpr int kBsaThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr uint32_t kBsaTmemCols = 512;
constexpr uint32_t kColS = 0;    // S/P buffers at columns 0 and 128
constexpr uint32_t kColO = 256;  // O accumulator, 128 columns
constexpr uint32_t kColQ = 384;  // Q (A operand of S = Q K^T): 64 columns bf16, 32 e4m3

template <bool kFp8>
struct BsaCfg {
  static constexpr int kTileBytes = kFp8 ? 16384 : 32768;  // one 128 x 128 K or V block
  static constexpr int kSlots = kFp8 ? 12 : 6;             // K/V ring (192 KB)
  static constexpr float kRescaleLog2 = kFp8 ? 1.f : 8.f;  // max growth before O is rescaled
  static constexpr float kPScale = kFp8 ? 224.f : 1.f;     // P multiplier before rounding (e4m3: 2 * 224 = 448)
};

template <bool kFp8>
struct BsaSmem {
  uint8_t ring[BsaCfg<kFp8>::kSlots][BsaCfg<kFp8>::kTileBytes];  // 1024-aligned
  uint64_t full[BsaCfg<kFp8>::kSlots];
  uint64_t empty[BsaCfg<kFp8>::kSlots];
  uint64_t q_ready;   // 8 softmax warps stored Q into TMEM
  uint64_t s_full[2];
  uint64_t p_full[2]; // 8 softmax warps stored P_n (and rescaled O if needed)
  uint64_t pv_done;   // one completion per P.V product
  uint64_t mx_full[2];// 8 softmax warps published their partial row maxima
  uint64_t sum_full;  // 8 softmax warps published their partial row sums
  uint64_t drain;     // completion of every MMA this CTA issued
  float pmax[2][2][128];  // [block parity][warpgroup][row] partial row maxima
  float psum[2][128];     // [warpgroup][row] partial row sums
  uint32_t tmem_base;
  int nvalid;         // valid entries of this CTA's list
  int abort;
};

// Next valid list entry at or after position p: 0 <= j <= i and strictly
// above the previous valid entry.  Every role applies the same rule, so all
// of them skip the same entries.  Returns the entry's position or `end`.
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

// Number of valid entries of a row, computed by one warp: a well-formed row
// (every entry in [0, i] and above its predecessor) is checked 32 entries at a
// time; only a malformed row is rescanned entry by entry.
__device__ __forceinline__ int count_valid_warp(const int32_t* __restrict__ col, int beg, int end, int i) {
  const int lane = lane_id();
  bool good = true;
  for (int p0 = beg; p0 < end; p0 += 32) {
    const int p = p0 + lane;
    const int j = p < end ? __ldg(col + p) : 0;
    int before = __shfl_up_sync(0xffffffffu, j, 1);
    if (lane == 0) before = p0 > beg ? __ldg(col + p0 - 1) : -1;
    const bool bad = p < end && (j < 0 || j > i || j <= before);
    if (__any_sync(0xffffffffu, bad)) { good = false; break; }
  }
  if (good) return end - beg;
  int n = 0, prev = -1, j = 0;
  for (int p = next_valid(col, beg, end, prev, i, &j); p < end; p = next_valid(col, p + 1, end, prev, i, &j)) {
    prev = j;
    ++n;
  }
  return n;
}

}  // namespace

template <bool kFp8>
__global__ void __launch_bounds__(kBsaThreads, 1)
    bsa_kernel(const __grid_constant__ BsaMaps maps, const SeqBatch batch, const BsaArgs args) {
  using Cfg = BsaCfg<kFp8>;
  constexpr int kSlots = Cfg::kSlots;
  extern __shared__ uint8_t smem_raw[];
  BsaSmem<kFp8>& sm =
      *reinterpret_cast<BsaSmem<kFp8>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = warp_id(), lane = lane_id();
  const int seq = find_seq(batch, blockIdx.x);
  const int local = blockIdx.x - batch.item0[seq];
  const int nb = batch.nb[seq];
  const int L = batch.len[seq];
  const int i = nb - 1 - local / args.hq;  // longest rows first
  const int h = local % args.hq;
  const int hk = h / (args.hq / args.hkv);
  const size_t r = static_cast<size_t>(h) * args.nbtot + batch.g0[seq] + i;
  const int pbeg = args.row_ptr[r];
  const int pend = args.row_ptr[r + 1];

  if (warp == kProducerWarp) {
    const int nv = count_valid_warp(args.col_idx, pbeg, pend, i);
    if (lane == 0) sm.nvalid = nv;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.q_ready, 8);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.p_full[b], 8);
    }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.mx_full[0], 8);
    mbar_init(&sm.mx_full[1], 8);
    mbar_init(&sm.sum_full, 8);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kBsaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int nvalid = sm.nvalid;
  volatile int* abort = &sm.abort;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nvalid > 0) {
      const CUtensorMap* mk = &maps.k[seq];
      const CUtensorMap* mv = &maps.v[seq];
      tma_prefetch_desc(mk);
      tma_prefetch_desc(mv);
      int j = 0, prev = -1;
      int t = 0;  // ring tile counter: K_n is tile 2n, V_n is tile 2n+1
      bool ok = true;
      for (int p = next_valid(args.col_idx, pbeg, pend, prev, i, &j); p < pend && ok;
           p = next_valid(args.col_idx, p + 1, pend, prev, i, &j)) {
        prev = j;
        for (int kv = 0; kv < 2; ++kv, ++t) {
          const int slot = t % kSlots;
          if (!mbar_wait(&sm.empty[slot], ((t / kSlots) & 1) ^ 1u, abort, args.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.full[slot], Cfg::kTileBytes);
          const CUtensorMap* m = kv == 0 ? mk : mv;
          for (int hh = 0; hh < (kFp8 ? 1 : 2); ++hh)
            tma_load_3d(sm.ring[slot] + hh * 16384, m, &sm.full[slot], hh * 64, hk, j * kBlock);
        }
      }
    }
    if (lane == 0 && nvalid != pend - pbeg) set_status(args.status, STEM_ERR_BAD_BLOCKLIST_CODE);
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nvalid > 0) {
      const uint32_t idesc_s = make_idesc(kFp8 ? 0u : 1u, 0u, 128u, 128u);
      const uint32_t idesc_o = make_idesc(kFp8 ? 0u : 1u, 1u, 128u, 128u);
      bool ok = mbar_wait(&sm.q_ready, 0, abort, args.status);
      tc_fence_after();
      for (int n = 0; n <= nvalid && ok; ++n) {
        if (n < nvalid) {  // S_n = Q K_n^T
          const int t = 2 * n, slot = t % kSlots;
          if (!mbar_wait(&sm.full[slot], (t / kSlots) & 1, abort, args.status)) break;
          tc_fence_after();
          const uint32_t sk = smem_u32(sm.ring[slot]);
          const uint32_t d_tmem = tmem + kColS + (n & 1) * 128;
          if constexpr (kFp8) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // 32 head dims per step
              mma_f8_ts(d_tmem, tmem + kColQ + kk * 8, make_sdesc_sw128(sk + kk * 32, 16, 1024), idesc_s, kk != 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 head dims per step
              mma_bf16_ts(d_tmem, tmem + kColQ + kk * 8,
                          make_sdesc_sw128(sk + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024), idesc_s, kk != 0);
          }
          mma_commit(&sm.s_full[n & 1]);
          mma_commit(&sm.empty[slot]);
        }
        if (n >= 1) {  // O += P_m V_m, m = n - 1
          const int m = n - 1;
          const int t = 2 * m + 1, slot = t % kSlots;
          if (!mbar_wait(&sm.p_full[m & 1], (m >> 1) & 1, abort, args.status)) break;
          if (!mbar_wait(&sm.full[slot], (t / kSlots) & 1, abort, args.status)) break;
          tc_fence_after();
          const uint32_t sv = smem_u32(sm.ring[slot]);
          const uint32_t p_tmem = tmem + kColS + (m & 1) * 128;
          if constexpr (kFp8) {
#pragma unroll
            for (int part = 0; part < 2; ++part)  // hi, then lo
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)      // 32 keys per step
                mma_f8_ts(tmem + kColO, p_tmem + part * 32 + kk * 8, make_sdesc_sw128(sv + kk * 4096, 16384, 1024),
                          idesc_o, (m | part | kk) != 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // 16 keys per step
              mma_bf16_ts(tmem + kColO, p_tmem + kk * 8, make_sdesc_sw128(sv + kk * 2048, 16384, 1024), idesc_o,
                          (m | kk) != 0);
          }
          mma_commit(&sm.pv_done);
          mma_commit(&sm.empty[slot]);
        }
      }
      // no MMA may still run when TMEM is released
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort, args.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int g = warp >> 2;      // column half
    const int q4 = warp & 3;      // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int t_row = i * kBlock + row;  // token of this row inside the sequence
    const size_t tok = static_cast<size_t>(batch.tok0[seq]) + t_row;
    float c = args.scale_log2;  // sigma * log2(e) (* q_scale * k_scale for fp8)
    if constexpr (kFp8) c *= args.q_scale[h] * args.k_scale[hk];
    const float ninf = -__int_as_float(0x7f800000);

    bool ok = true;
    if (nvalid > 0) {
      // Q row half -> TMEM (A operand of S = Q K^T); rows past the sequence end are zero
      constexpr int kRowBytes = kFp8 ? 128 : 256;
      const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(args.q) +
                                                        (tok * args.hq + h) * kRowBytes + g * (kRowBytes / 2));
      if constexpr (kFp8) {
        uint32_t w[16];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const uint4 v = t_row < L ? __ldg(src + x) : make_uint4(0, 0, 0, 0);
          w[4 * x] = v.x; w[4 * x + 1] = v.y; w[4 * x + 2] = v.z; w[4 * x + 3] = v.w;
        }
        tmem_st16(tmem + kColQ + 16 * g + lane_off, w);
      } else {
        uint32_t w[32];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const uint4 v = t_row < L ? __ldg(src + x) : make_uint4(0, 0, 0, 0);
          w[4 * x] = v.x; w[4 * x + 1] = v.y; w[4 * x + 2] = v.z; w[4 * x + 3] = v.w;
        }
        tmem_st32(tmem + kColQ + 32 * g + lane_off, w);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.q_ready);
    }

    float m_ref = ninf;  // reference max (scaled log2 domain) shared by O and the sums
    float l = 0.f;       // partial row sum of exp over this warpgroup's columns
    int pv_seen = 0;     // P.V completions consumed
    auto wait_pv = [&](int upto) -> bool {  // until PV_0 .. PV_upto are complete
      while (pv_seen <= upto) {
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done, pv_seen & 1, abort, args.status))) return false;
        ++pv_seen;
      }
      return true;
    };

    int j = 0, prev = -1;
    int p = next_valid(args.col_idx, pbeg, pend, prev, i, &j);
    for (int n = 0; n < nvalid; ++n) {
      const int b = n & 1;
      const bool diag = (j == i);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[b], (n >> 1) & 1, abort, args.status))) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_addr = tmem + kColS + b * 128 + lane_off;
      float sv[64];
      {
        uint32_t rr[32];
        tmem_ld32(s_addr + 64 * g, rr);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) sv[x] = __uint_as_float(rr[x]);
        tmem_ld32(s_addr + 64 * g + 32, rr);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) sv[32 + x] = __uint_as_float(rr[x]);
      }
      if (diag) {
#pragma unroll
        for (int x = 0; x < 64; ++x)
          if (64 * g + x > row) sv[x] = ninf;
      }
      float mx = ninf;
#pragma unroll
      for (int x = 0; x < 64; ++x) mx = fmaxf(mx, sv[x]);
      sm.pmax[b][g][row] = mx;
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.mx_full[b]);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.mx_full[b], (n >> 1) & 1, abort, args.status))) { ok = false; break; }
      mx = fmaxf(mx, sm.pmax[b][g ^ 1][row]);
      // move the reference only when the max grew past the threshold
      const float m_cand = mx * c;
      const bool need = (m_ref == ninf) ? (m_cand != ninf) : (m_cand > m_ref + Cfg::kRescaleLog2);
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = need ? m_cand : m_ref;
        const float alpha = (m_ref == ninf) ? 0.f : fast_exp2(m_ref - m_new);
        l *= alpha;
        if (n >= 1) {
          if (!wait_pv(n - 1)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int hc = 0; hc < 2; ++hc) {
            const uint32_t oa = tmem + kColO + 64 * g + 32 * hc + lane_off;
            uint32_t rr[32];
            tmem_ld32(oa, rr);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < 32; ++x) rr[x] = __float_as_uint(__uint_as_float(rr[x]) * alpha);
            tmem_st32(oa, rr);
          }
          tmem_st_wait();
        }
        m_ref = m_new;
      }
      // probabilities p = exp2(s c - m_ref), written over S as the A operand of P.V
      const float m_use = (m_ref == ninf) ? 0.f : m_ref;
      const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_use, -m_use);
      float psum = 0.f;
      if constexpr (kFp8) {
        uint32_t whi[16], wlo[16];
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          const float2 a = ffma2(make_float2(sv[4 * x], sv[4 * x + 1]), c2, nm2);
          const float2 a2 = ffma2(make_float2(sv[4 * x + 2], sv[4 * x + 3]), c2, nm2);
          const float p0 = fast_exp2(a.x), p1 = fast_exp2(a.y), p2 = fast_exp2(a2.x), p3 = fast_exp2(a2.y);
          psum += (p0 + p1) + (p2 + p3);
          const uint32_t x01 = f32x2_to_f16x2(p0 * Cfg::kPScale, p1 * Cfg::kPScale);
          const uint32_t x23 = f32x2_to_f16x2(p2 * Cfg::kPScale, p3 * Cfg::kPScale);
          const uint16_t h01 = f16x2_to_e4m3x2(x01), h23 = f16x2_to_e4m3x2(x23);
          const uint16_t l01 = f16x2_to_e4m3x2(hsub2_u32(x01, e4m3x2_to_f16x2(h01)));
          const uint16_t l23 = f16x2_to_e4m3x2(hsub2_u32(x23, e4m3x2_to_f16x2(h23)));
          whi[x] = static_cast<uint32_t>(h01) | (static_cast<uint32_t>(h23) << 16);
          wlo[x] = static_cast<uint32_t>(l01) | (static_cast<uint32_t>(l23) << 16);
        }
        tmem_st16(tmem + kColS + b * 128 + 16 * g + lane_off, whi);
        tmem_st16(tmem + kColS + b * 128 + 32 + 16 * g + lane_off, wlo);
      } else {
        uint32_t w[32];
#pragma unroll
        for (int x = 0; x < 32; ++x) {
          const float2 a = ffma2(make_float2(sv[2 * x], sv[2 * x + 1]), c2, nm2);
          const float p0 = fast_exp2(a.x), p1 = fast_exp2(a.y);
          psum += p0 + p1;
          w[x] = pack_bf16x2(p0, p1);
        }
        tmem_st32(tmem + kColS + b * 128 + 32 * g + lane_off, w);
      }
      l += psum;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.p_full[b]);
      // keep the P.V completions consumed in step (normally already complete)
      if (n >= 1 && !wait_pv(n - 1)) { ok = false; break; }
      prev = j;
      p = next_valid(args.col_idx, p + 1, pend, prev, i, &j);
    }

    // epilogue: combine the two halves' row sums, normalise O, store
    float o[64];
#pragma unroll
    for (int x = 0; x < 64; ++x) o[x] = 0.f;
    if (ok && nvalid > 0 && wait_pv(nvalid - 1)) {
      tc_fence_after();
#pragma unroll
      for (int hc = 0; hc < 2; ++hc) {
        uint32_t rr[32];
        tmem_ld32(tmem + kColO + 64 * g + 32 * hc + lane_off, rr);
        tmem_ld_wait();
#pragma unroll
        for (int x = 0; x < 32; ++x) o[32 * hc + x] = __uint_as_float(rr[x]);
      }
    }
    sm.psum[g][row] = l;
    __syncwarp();
    if (lane == 0) mbar_arrive(&sm.sum_full);
    const bool sums_ok = __all_sync(0xffffffffu, mbar_wait(&sm.sum_full, 0, abort, args.status));
    const float l_tot = sums_ok ? l + sm.psum[g ^ 1][row] : 0.f;
    if (t_row < L) {
      float inv = (l_tot > 0.f) ? 1.f / l_tot : 0.f;
      if constexpr (kFp8) inv *= args.v_scale[hk] * (1.f / Cfg::kPScale);
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                            (tok * args.hq + h) * static_cast<size_t>(kHeadDim) * 2 + g * 128);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(o[q * 8 + e * 2] * inv, o[q * 8 + e * 2 + 1] * inv);
        dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (g == 0) {
        const float lse = (l_tot > 0.f) ? (m_ref + __log2f(l_tot)) * 0.69314718055994530942f : ninf;
        args.lse[static_cast<size_t>(h) * args.total_tokens + tok] = lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kBsaTmemCols);
  }
}

size_t bsa_smem_bytes(bool fp8) { return (fp8 ? sizeof(BsaSmem<true>) : sizeof(BsaSmem<false>)) + 1024; }

cudaError_t launch_bsa(const BsaMaps& maps, const SeqBatch& batch, const BsaArgs& args, bool fp8,
                       cudaStream_t stream) {
  const int items = batch.item0[batch.n];
  if (items == 0) return cudaSuccess;
  const size_t smem = bsa_smem_bytes(fp8);
  cudaError_t e;
  if (fp8) {
    e = cudaFuncSetAttribute(bsa_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bsa_kernel<true><<<items, kBsaThreads, smem, stream>>>(maps, batch, args);
  } else {
    e = cudaFuncSetAttribute(bsa_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bsa_kernel<false><<<items, kBsaThreads, smem, stream>>>(maps, batch, args);
  }
  return cudaGetLastError();
}

}  // namespace stem
