// k_bsa.cu — causal block-sparse flash attention over pre-compacted block lists.
//
// "Stem" gist.science zh §2.3 (exact softmax and aggregation only over the
// selected blocks); youleyou HPC-BSA article §3.1 (the inner loop walks a list
// prepared outside it; a skipped block is the same as a block of -inf scores,
// so the softmax needs no change; fixed 128 x 128 tiles).
//
// One CTA owns one CSR row: a 128-token query block of one query head.  For
// every listed key block j (ascending, the diagonal last):
//   S = Q K_j^T            tcgen05.mma, fp32 in TMEM (two S buffers)
//   P = exp2(S c - m)      softmax warps, online max/sum in fp32, causal mask
//                          only when j is the diagonal block
//   O_j = P V_j            tcgen05.mma with P staged 128-B swizzled in SMEM
//                          (bf16, or e4m3 scaled by 448 for the fp8 path)
//   o = (o + O_{j-1}) a_j  rescale-and-accumulate in registers
// K and V blocks arrive by TMA (per-sequence tensor maps, so reads past the
// sequence end are zero-filled) into a two-stage ring.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2-5 softmax/epilogue (thread = query row = TMEM lane).
#include "stem_device.cuh"
#include "stem_kernels.h"

namespace stem {

namespace {

constexpr int kBsaThreads = 192;
constexpr uint32_t kBsaTmemCols = 512;  // S0, S1, O0, O1 (128 columns each)

template <bool kFp8>
struct BsaCfg {
  static constexpr int kRowBytes = kFp8 ? 128 : 256;       // one token row of d = 128
  static constexpr int kTileBytes = 128 * kRowBytes;       // 128 x 128 tile
  static constexpr int kHalf = 16384;                      // one 128 x 128-B swizzled slab
};

template <bool kFp8>
struct BsaSmem {
  uint8_t q[BsaCfg<kFp8>::kTileBytes];
  uint8_t k[2][BsaCfg<kFp8>::kTileBytes];
  uint8_t v[2][BsaCfg<kFp8>::kTileBytes];
  uint8_t p[2][BsaCfg<kFp8>::kTileBytes];
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2];
  uint64_t v_full[2], v_empty[2];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full[2], p_empty[2];
  uint64_t o_full[2], o_empty[2];
  uint64_t drain;  // completion of every MMA this CTA issued
  uint32_t tmem_base;
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

}  // namespace

template <bool kFp8>
__global__ void __launch_bounds__(kBsaThreads, 1)
    bsa_kernel(const __grid_constant__ BsaMaps maps, const SeqBatch batch, const BsaArgs args) {
  using Cfg = BsaCfg<kFp8>;
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

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.k_full[b], 1);
      mbar_init(&sm.k_empty[b], 1);
      mbar_init(&sm.v_full[b], 1);
      mbar_init(&sm.v_empty[b], 1);
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_empty[b], 4);
      mbar_init(&sm.p_full[b], 4);
      mbar_init(&sm.p_empty[b], 1);
      mbar_init(&sm.o_full[b], 1);
      mbar_init(&sm.o_empty[b], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kBsaTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      const CUtensorMap* mq = &maps.q[seq];
      const CUtensorMap* mk = &maps.k[seq];
      const CUtensorMap* mv = &maps.v[seq];
      int j, prev = -1;
      int p = next_valid(args.col_idx, pbeg, pend, prev, i, &j);
      // report malformed entries once
      for (int pp = pbeg, pv = -1; pp < pend; ++pp) {
        const int jj = __ldg(args.col_idx + pp);
        if (jj >= 0 && jj <= i && jj > pv) pv = jj;
        else { set_status(args.status, STEM_ERR_BAD_BLOCKLIST_CODE); break; }
      }
      if (p < pend) {
        tma_prefetch_desc(mq);
        tma_prefetch_desc(mk);
        tma_prefetch_desc(mv);
        mbar_arrive_expect_tx(&sm.q_full, Cfg::kTileBytes);
        for (int hh = 0; hh < (kFp8 ? 1 : 2); ++hh)
          tma_load_3d(sm.q + hh * Cfg::kHalf, mq, &sm.q_full, hh * 64, h, i * kBlock);
      }
      for (int n = 0; p < pend; ++n) {
        const int st = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        if (!mbar_wait(&sm.k_empty[st], ph ^ 1u, abort, args.status)) break;
        mbar_arrive_expect_tx(&sm.k_full[st], Cfg::kTileBytes);
        for (int hh = 0; hh < (kFp8 ? 1 : 2); ++hh)
          tma_load_3d(sm.k[st] + hh * Cfg::kHalf, mk, &sm.k_full[st], hh * 64, hk, j * kBlock);
        if (!mbar_wait(&sm.v_empty[st], ph ^ 1u, abort, args.status)) break;
        mbar_arrive_expect_tx(&sm.v_full[st], Cfg::kTileBytes);
        for (int hh = 0; hh < (kFp8 ? 1 : 2); ++hh)
          tma_load_3d(sm.v[st] + hh * Cfg::kHalf, mv, &sm.v_full[st], hh * 64, hk, j * kBlock);
        prev = j;
        p = next_valid(args.col_idx, p + 1, pend, prev, i, &j);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc(kFp8 ? 0u : 1u, 0u, 128u, 128u);
      const uint32_t idesc_o = make_idesc(kFp8 ? 0u : 1u, 1u, 128u, 128u);
      int j, prev = -1;
      int p = next_valid(args.col_idx, pbeg, pend, prev, i, &j);
      bool ok = true;
      if (p < pend) ok = mbar_wait(&sm.q_full, 0, abort, args.status);
      auto issue_pv = [&](int m) -> bool {
        const int st = m & 1;
        const uint32_t ph = (m >> 1) & 1;
        if (!mbar_wait(&sm.v_full[st], ph, abort, args.status)) return false;
        if (!mbar_wait(&sm.p_full[st], ph, abort, args.status)) return false;
        if (!mbar_wait(&sm.o_empty[st], ph ^ 1u, abort, args.status)) return false;
        tc_fence_after();
        const uint32_t sp = smem_u32(sm.p[st]);
        const uint32_t sv = smem_u32(sm.v[st]);
        const uint32_t d_tmem = tmem + 256 + st * 128;
        if constexpr (kFp8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 32 keys per step
            mma_f8_ss(d_tmem, make_sdesc_sw128(sp + kk * 32, 16, 1024),
                      make_sdesc_sw128(sv + kk * 4096, 16384, 1024), idesc_o, kk != 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // 16 keys per step
            mma_bf16_ss(d_tmem, make_sdesc_sw128(sp + (kk >> 2) * Cfg::kHalf + (kk & 3) * 32, 16, 1024),
                        make_sdesc_sw128(sv + kk * 2048, Cfg::kHalf, 1024), idesc_o, kk != 0);
        }
        mma_commit(&sm.o_full[st]);
        mma_commit(&sm.v_empty[st]);
        mma_commit(&sm.p_empty[st]);
        return true;
      };
      int n = 0;
      for (; p < pend && ok; ++n) {
        const int st = n & 1;
        const uint32_t ph = (n >> 1) & 1;
        if (!mbar_wait(&sm.k_full[st], ph, abort, args.status)) { ok = false; break; }
        if (!mbar_wait(&sm.s_empty[st], ph ^ 1u, abort, args.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sq = smem_u32(sm.q);
        const uint32_t sk = smem_u32(sm.k[st]);
        const uint32_t d_tmem = tmem + st * 128;
        if constexpr (kFp8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_f8_ss(d_tmem, make_sdesc_sw128(sq + kk * 32, 16, 1024), make_sdesc_sw128(sk + kk * 32, 16, 1024),
                      idesc_s, kk != 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * Cfg::kHalf + (kk & 3) * 32;
            mma_bf16_ss(d_tmem, make_sdesc_sw128(sq + off, 16, 1024), make_sdesc_sw128(sk + off, 16, 1024),
                        idesc_s, kk != 0);
          }
        }
        mma_commit(&sm.s_full[st]);
        mma_commit(&sm.k_empty[st]);
        if (n >= 1 && !issue_pv(n - 1)) { ok = false; break; }
        prev = j;
        p = next_valid(args.col_idx, p + 1, pend, prev, i, &j);
      }
      if (ok && n >= 1) issue_pv(n - 1);
      // no MMA may still run when TMEM is released
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort, args.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int t = i * kBlock + row;  // token of this row inside the sequence
    float c = args.scale_log2;       // sigma * log2(e) (* q_scale * k_scale for fp8)
    if constexpr (kFp8) c *= args.q_scale[h] * args.k_scale[hk];
    const float ninf = -__int_as_float(0x7f800000);
    float m_run = ninf, l_run = 0.f;
    float o[128];
#pragma unroll
    for (int x = 0; x < 128; ++x) o[x] = 0.f;
    int j, prev = -1;
    int p = next_valid(args.col_idx, pbeg, pend, prev, i, &j);
    int n = 0;
    bool ok = true;
    for (; p < pend; ++n) {
      const int st = n & 1;
      const uint32_t ph = (n >> 1) & 1;
      const bool diag = (j == i);
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[st], ph, abort, args.status))) { ok = false; break; }
      tc_fence_after();
      const uint32_t s_addr = tmem + st * 128 + lane_off;
      // pass 1: row max of the raw logits
      float mx = ninf;
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rr[32];
        tmem_ld32(s_addr + ch * 32, rr);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const bool masked = diag && (ch * 32 + cc > row);
          mx = masked ? mx : fmaxf(mx, __uint_as_float(rr[cc]));
        }
      }
      const float m_new = fmaxf(m_run, mx * c);
      const float m_use = (m_new == ninf) ? 0.f : m_new;
      const float alpha = fast_exp2(m_run - m_use);
      // pass 2: probabilities, staged to SMEM as the A operand of P.V
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.p_empty[st], ph ^ 1u, abort, args.status))) { ok = false; break; }
      float rowsum = 0.f;
      uint8_t* prow = sm.p[st];
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rr[32];
        tmem_ld32(s_addr + ch * 32, rr);
        tmem_ld_wait();
        float pv[32];
#pragma unroll
        for (int cc = 0; cc < 32; ++cc) {
          const bool masked = diag && (ch * 32 + cc > row);
          pv[cc] = masked ? 0.f : fast_exp2(fmaf(__uint_as_float(rr[cc]), c, -m_use));
          rowsum += pv[cc];
        }
        if constexpr (kFp8) {
          // 32 keys -> 32 bytes = two 16-byte chunks of the 128-byte row
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint16_t lo = pack_e4m3x2(pv[q * 16 + e * 4 + 0] * 448.f, pv[q * 16 + e * 4 + 1] * 448.f);
              const uint16_t hi = pack_e4m3x2(pv[q * 16 + e * 4 + 2] * 448.f, pv[q * 16 + e * 4 + 3] * 448.f);
              w[e] = static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
            }
            const int chunk = (ch * 2 + q) ^ (row & 7);
            *reinterpret_cast<uint4*>(prow + row * 128 + chunk * 16) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          // 32 keys -> 64 bytes = four 16-byte chunks; 64 keys per 128-byte slab
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(pv[q * 8 + e * 2], pv[q * 8 + e * 2 + 1]);
            const int chunk = ((ch & 1) * 4 + q) ^ (row & 7);
            *reinterpret_cast<uint4*>(prow + (ch >> 1) * Cfg::kHalf + row * 128 + chunk * 16) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      l_run = l_run * alpha + rowsum;
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.p_full[st]);
        mbar_arrive(&sm.s_empty[st]);
      }
      // fold in the previous block's P.V (relative to m_run) and rescale to m_new
      if (n >= 1) {
        const int so = (n - 1) & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full[so], ((n - 1) >> 1) & 1, abort, args.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t rr[32];
          tmem_ld32(tmem + 256 + so * 128 + lane_off + ch * 32, rr);
          tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) o[ch * 32 + cc] = (o[ch * 32 + cc] + __uint_as_float(rr[cc])) * alpha;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.o_empty[so]);
      }
      m_run = m_new;
      prev = j;
      p = next_valid(args.col_idx, p + 1, pend, prev, i, &j);
    }
    if (ok && n >= 1) {
      const int so = (n - 1) & 1;
      if (__all_sync(0xffffffffu, mbar_wait(&sm.o_full[so], ((n - 1) >> 1) & 1, abort, args.status))) {
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t rr[32];
          tmem_ld32(tmem + 256 + so * 128 + lane_off + ch * 32, rr);
          tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) o[ch * 32 + cc] += __uint_as_float(rr[cc]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.o_empty[so]);
      } else {
        ok = false;
      }
    }
    // epilogue: normalise and store this row
    if (t < L) {
      float inv = (l_run > 0.f) ? 1.f / l_run : 0.f;
      if constexpr (kFp8) inv *= args.v_scale[hk] * (1.f / 448.f);
      const size_t tok = static_cast<size_t>(batch.tok0[seq]) + t;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                            (tok * args.hq + h) * static_cast<size_t>(kHeadDim) * 2);
#pragma unroll
      for (int q = 0; q < 16; ++q) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = pack_bf16x2(o[q * 8 + e * 2] * inv, o[q * 8 + e * 2 + 1] * inv);
        dst[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
      const float lse = (l_run > 0.f) ? (m_run + __log2f(l_run)) * 0.69314718055994530942f : ninf;
      args.lse[static_cast<size_t>(h) * args.total_tokens + tok] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
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
