// k_bsa_pair.cu — block-sparse attention for block lists shared by the query
// heads of a KV group.
//
// "Stem" gist.science zh §2.3 (exact softmax over the selected blocks);
// youleyou HPC-BSA article §3.1 (compacted lists walked by the inner loop) and
// §4 (one block list per KV group, so a K/V tile staged once serves several
// query heads).
//
// With shared lists (STEM_LIST_PER_GROUP) the rows (i, h) and (i, h + 1) of
// two query heads of one KV group walk the same key blocks, so one CTA owns
// both rows ("tiles") and stages every K and V half once for the two.  Per
// tile everything is as in the one-row kernel (k_bsa.cu): 64-key halves,
// double-buffered S in TMEM, P written over S, O accumulated in TMEM, lazy
// reference max.  Each tile has its softmax warpgroup and its MMA issuer; the
// K and V producers are shared, so a K slot is reused once both tiles' S_h
// are complete and a V slot once both tiles' P_h V_h are.
//
// Warp roles (384 threads):
//   warps 0-3    softmax + epilogue of tile 0 (TMEM lane quarters 0-3)
//   warps 4-7    softmax + epilogue of tile 1
//   warp  8      TMA producer of both Q blocks and the K halves (stages the list)
//   warp  9      TMA producer of the V halves (checks the two rows' lists agree)
//   warps 10, 11 MMA issuer of tile 0, 1 (warp 10 owns the TMEM allocation)
// One CTA per SM (all 512 TMEM columns: tile t has S buffers at 256 t and
// 256 t + 64 and O at 256 t + 128).  An odd group leaves the last pair with
// one tile.  Every wait is bounded.
#include "stem_bsa_common.cuh"

namespace stem {

namespace {

constexpr int kPairThreads = 384;
constexpr int kPairKWarp = 8;
constexpr int kPairVWarp = 9;
constexpr int kPairMmaWarp = 10;  // + tile; warp 10 owns TMEM
constexpr uint32_t kPairTmemCols = 512;

template <bool kFp8>
struct PairSmem {
  uint8_t q[2][BsaCfg<kFp8>::kQBytes];      // per tile; 1024-aligned
  uint8_t k[2][BsaCfg<kFp8>::kKHalfBytes];  // per slot, shared by the tiles
  uint8_t v[2][BsaCfg<kFp8>::kVHalfBytes];
  uint64_t q_full;        // both tiles' Q landed
  uint64_t k_full[2];     // per slot: K_h landed
  uint64_t v_full[2];     // per slot: V_h landed
  uint64_t s_full[2][2];  // per tile and S buffer: S_h complete
  uint64_t v_free[2][2];  // per tile and slot: P_h V_h complete
  uint64_t p_full[2][2];  // per tile and S buffer: the 4 softmax warps stored P_h
  uint64_t o_done[2];     // per tile: the last P V is complete
  uint64_t drain[2];      // per tile: every MMA of that tile's issuer complete
  int32_t list[kMaxList];
  int nvalid;
  int in_smem;
  uint32_t tmem_base;
  int abort;
};

// The two rows' lists are equal entry by entry (one warp).
__device__ bool lists_equal(const int32_t* __restrict__ col, const Tile& a, const Tile& b) {
  if (a.end - a.beg != b.end - b.beg) return false;
  const int lane = lane_id();
  bool same = true;
  for (int p0 = 0; p0 < a.end - a.beg && same; p0 += 32) {
    const int p = p0 + lane;
    const bool d = p < a.end - a.beg && __ldg(col + a.beg + p) != __ldg(col + b.beg + p);
    same = !__any_sync(0xffffffffu, d);
  }
  return same;
}

}  // namespace

template <bool kFp8>
__global__ void __launch_bounds__(kPairThreads, 1)
    bsa_pair_kernel(const __grid_constant__ BsaMaps maps, const SeqBatch batch, const BsaArgs args) {
  using Cfg = BsaCfg<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  PairSmem<kFp8>& sm =
      *reinterpret_cast<PairSmem<kFp8>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = warp_id(), lane = lane_id();
  const int seq = find_seq(batch, blockIdx.x);
  const int nb = batch.nb[seq];
  const int L = batch.len[seq];
  const int G = args.hq / args.hkv;
  const int npair = (G + 1) / 2;
  // CTAs of a sequence in KV-head-major order: KV head, then query blocks
  // descending (longest rows first), then the head pairs of the group
  Tile tile[2];
  {
    const int it = blockIdx.x - batch.item0[seq];
    const int hk_of = args.hk0 + it / (npair * nb);
    const int rem = it % (npair * nb);
    const int i = nb - 1 - rem / npair;
    const int pr = rem % npair;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      tile[t].valid = 2 * pr + t < G;
      tile[t].i = i;
      tile[t].h = hk_of * G + 2 * pr + (tile[t].valid ? t : 0);
      tile[t].hk = hk_of;
      const size_t r = static_cast<size_t>(tile[t].h) * args.nbtot + batch.g0[seq] + i;
      tile[t].beg = tile[t].valid ? args.row_ptr[r] : 0;
      tile[t].end = tile[t].valid ? args.row_ptr[r + 1] : 0;
    }
  }
  const bool two = tile[1].valid;

  if (warp == kPairKWarp) stage_list(args.col_idx, tile[0], sm.list, &sm.nvalid, &sm.in_smem, args.status);
  if (warp == kPairVWarp && two && !lists_equal(args.col_idx, tile[0], tile[1]) && lane == 0)
    set_status(args.status, STEM_ERR_BAD_BLOCKLIST_CODE);  // the second row is computed with the first's list
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.k_full[b], 1);
      mbar_init(&sm.v_full[b], 1);
      for (int t = 0; t < 2; ++t) {
        mbar_init(&sm.s_full[t][b], 1);
        mbar_init(&sm.v_free[t][b], 1);
        mbar_init(&sm.p_full[t][b], 4);
      }
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.o_done[t], 1);
      mbar_init(&sm.drain[t], 1);
    }
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kPairMmaWarp) {
    tmem_alloc(&sm.tmem_base, kPairTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const int N = sm.nvalid;
  const bool list_in_smem = sm.in_smem != 0;
  volatile int* abort = &sm.abort;
  const int ntiles = two ? 2 : 1;

  if (warp == kPairKWarp || warp == kPairVWarp) {
    // ------------------------------------------------------------ producers (shared)
    const bool is_v = warp == kPairVWarp;
    if (lane == 0 && N > 0) {
      // fp8 V is read from its packed f16 copy, which the widening pass
      // gathered through the page table
      const bool paged = args.page_table != nullptr && !(kFp8 && is_v);
      const CUtensorMap* m = paged ? (is_v ? &maps.v_pool : &maps.k_pool) : (is_v ? &maps.v[seq] : &maps.k[seq]);
      const int slabs = is_v ? 2 : Cfg::kKSlabs;
      const int half_bytes = is_v ? Cfg::kVHalfBytes : Cfg::kKHalfBytes;
      const int32_t* pages = paged ? args.page_table + static_cast<size_t>(batch.seq_id[seq]) * args.max_pages : nullptr;
      tma_prefetch_desc(m);
      if (!is_v) {
        mbar_arrive_expect_tx(&sm.q_full, ntiles * Cfg::kQBytes);
        for (int t = 0; t < ntiles; ++t)
          for (int sl = 0; sl < Cfg::kKSlabs; ++sl)
            tma_load_3d(sm.q[t] + sl * 16384, &maps.q[seq], &sm.q_full, sl * 64, tile[t].h, tile[t].i * kBlock);
      }
      const int H = 2 * N;
      ListCursor cur(tile[0].beg);
      int j = 0, issued = 0;
      for (int h = 0; h < H; ++h) {
        if (h >= 2) {
          // slot h % 2 is free once every tile's S_{h-2} (K) or P_{h-2}
          // V_{h-2} (V) is complete
          bool ok = true;
          for (int t = 0; t < ntiles && ok; ++t)
            ok = mbar_wait(is_v ? &sm.v_free[t][h & 1] : &sm.s_full[t][h & 1], ((h - 2) >> 1) & 1, abort,
                           args.status);
          if (!ok) break;
        }
        if ((h & 1) == 0) j = cur.next(sm.list, list_in_smem, h >> 1, args.col_idx, tile[0].end, tile[0].i);
        uint8_t* dst = is_v ? sm.v[h & 1] : sm.k[h & 1];
        uint64_t* bar = is_v ? &sm.v_full[h & 1] : &sm.k_full[h & 1];
        // token row of the half: in the sequence, or through the page table (a
        // 64-key half never straddles a page; a page number outside the pool
        // reads zeros)
        int row = j * kBlock + (h & 1) * kHalf;
        if (paged) row = __ldg(pages + row / args.page_size) * args.page_size + row % args.page_size;
        mbar_arrive_expect_tx(bar, half_bytes);
        for (int sl = 0; sl < slabs; ++sl) tma_load_3d(dst + sl * (kHalf * 128), m, bar, sl * 64, tile[0].hk, row);
        ++issued;
      }
      // every copy of this producer has landed before the CTA can exit
      if (!is_v) mbar_wait_quiesce(&sm.q_full, 0, args.status);
      for (int x = 0; x < 2 && x < issued; ++x) {
        const int last = issued - 1 - ((issued - 1 - x) & 1);  // last half issued into slot x
        mbar_wait_quiesce(is_v ? &sm.v_full[x] : &sm.k_full[x], (last >> 1) & 1, args.status);
      }
    }
    __syncwarp();
  } else if (warp >= kPairMmaWarp) {
    // ------------------------------------------------------------ MMA issuer of tile t
    const int t = warp - kPairMmaWarp;
    if (lane == 0 && N > 0 && t < ntiles) {
      const uint32_t idesc_s = make_idesc(kFp8 ? 0u : 1u, 0u, 128u, static_cast<uint32_t>(kHalf));
      const uint32_t idesc_o = make_idesc(kFp8 ? 0u : 1u, 1u, 128u, 128u);  // kind::f16: f16 (0) or bf16 (1)
      const uint32_t sq = smem_u32(sm.q[t]);
      const uint32_t base = tmem + 256 * t;
      const uint32_t o_tmem = base + 128;
      const int H = 2 * N;
      auto issue_s = [&](int h) -> bool {  // S_h = Q K_h^T into buffer h % 2 of the tile
        if (!mbar_wait(&sm.k_full[h & 1], (h >> 1) & 1, abort, args.status)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(sm.k[h & 1]);
        const uint32_t d = base + kHalf * (h & 1);
        if constexpr (kFp8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 32 head dims per step
            mma_f8_ss(d, make_sdesc_sw128(sq + kk * 32, 16, 1024), make_sdesc_sw128(sk + kk * 32, 16, 1024), idesc_s,
                      kk != 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)  // 16 head dims per step
            mma_bf16_ss(d, make_sdesc_sw128(sq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                        make_sdesc_sw128(sk + (kk >> 2) * (kHalf * 128) + (kk & 3) * 32, 16, 1024), idesc_s, kk != 0);
        }
        mma_commit(&sm.s_full[t][h & 1]);
        return true;
      };
      auto issue_pv = [&](int h) -> bool {  // O += P_h V_h (kind::f16: bf16, or f16 on the fp8 path)
        if (!mbar_wait(&sm.p_full[t][h & 1], (h >> 1) & 1, abort, args.status)) return false;
        if (!mbar_wait(&sm.v_full[h & 1], (h >> 1) & 1, abort, args.status)) return false;
        tc_fence_after();
        const uint32_t sv = smem_u32(sm.v[h & 1]);
        const uint32_t p = base + kHalf * (h & 1);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 keys per step
          mma_bf16_ts(o_tmem, p + kk * 8, make_sdesc_sw128(sv + kk * 2048, kHalf * 128, 1024), idesc_o,
                      (h | kk) != 0);
        mma_commit(&sm.v_free[t][h & 1]);
        if (h == H - 1) mma_commit(&sm.o_done[t]);
        return true;
      };
      // S_0, S_1, then per half h: P_h V_h and S_{h+2} (into the buffer P_h
      // V_h just read: one issuer's products run in order)
      bool ok = mbar_wait(&sm.q_full, 0, abort, args.status) && issue_s(0) && issue_s(1);
      for (int h = 0; h < H && ok; ++h) {
        ok = issue_pv(h);
        if (ok && h + 2 < H) ok = issue_s(h + 2);
      }
      // no MMA of this issuer may still run when TMEM is released
      mma_commit(&sm.drain[t]);
      mbar_wait_quiesce(&sm.drain[t], 0, args.status);
    }
    __syncwarp();
  } else if ((warp >> 2) < ntiles) {
    // ------------------------------------------------------------ softmax + epilogue of tile t
    const int t = warp >> 2;
    const int q4 = warp & 3;  // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const Tile tl = (t == 0) ? tile[0] : tile[1];  // per-field selects, no local-memory indexing
    const int t_row = tl.i * kBlock + row;        // token of this row inside the sequence
    const size_t tok = static_cast<size_t>(batch.tok0[seq]) + t_row;
    float c = args.scale_log2;  // sigma * log2(e) (* q_scale * k_scale for fp8)
    if constexpr (kFp8) c *= args.q_scale[tl.h] * args.k_scale[tl.hk];
    const float ninf = -__int_as_float(0x7f800000);
    const uint32_t s_base = tmem + 256 * t + lane_off;
    const uint32_t o_tmem = tmem + 256 * t + 128 + lane_off;

    float m_ref = ninf;  // reference max (scaled log2 domain) shared by O and l
    float l = 0.f;       // row sum of exp2(s c - m_ref)
    bool ok = true;
    ListCursor cur(tile[0].beg);
    for (int n = 0; n < N && ok; ++n) {
      const int j = cur.next(sm.list, list_in_smem, n, args.col_idx, tile[0].end, tl.i);
      const bool diag = (j == tl.i);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        const int h = 2 * n + half;
        const uint32_t s_tmem = s_base + kHalf * half;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[t][half], n & 1, abort, args.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        // the half's 64 scores, loaded once and kept in registers
        uint32_t rr[2][32];
        tmem_ld32(s_tmem, rr[0]);
        tmem_ld32(s_tmem + 32, rr[1]);
        tmem_ld_wait();
        if (diag) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (half * kHalf + ch * 32 + x > row) rr[ch][x] = 0xff800000u;  // -inf -> p = 0
        }
        float m4[4];
#pragma unroll
        for (int a = 0; a < 4; ++a)
          m4[a] = fmax3(__uint_as_float(rr[a >> 1][(a & 1) * 16]), __uint_as_float(rr[a >> 1][(a & 1) * 16 + 1]),
                        __uint_as_float(rr[a >> 1][(a & 1) * 16 + 2]));
#pragma unroll
        for (int x = 3; x < 15; x += 2)
#pragma unroll
          for (int a = 0; a < 4; ++a)
            m4[a] = fmax3(m4[a], __uint_as_float(rr[a >> 1][(a & 1) * 16 + x]),
                          __uint_as_float(rr[a >> 1][(a & 1) * 16 + x + 1]));
#pragma unroll
        for (int a = 0; a < 4; ++a) m4[a] = fmaxf(m4[a], __uint_as_float(rr[a >> 1][(a & 1) * 16 + 15]));
        const float m_cand = fmax3(m4[0], m4[1], fmaxf(m4[2], m4[3])) * c;
        // move the reference only when the max grew past the threshold
        const bool need = (m_ref == ninf) ? (m_cand != ninf) : (m_cand > m_ref + Cfg::kRescaleLog2);
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = need ? m_cand : m_ref;
          const float alpha = (m_ref == ninf) ? 0.f : fast_exp2(m_ref - m_new);
          l *= alpha;
          if (h >= 1) {
            // O holds P V up to half h-1: let that product finish first
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&sm.v_free[t][(h - 1) & 1], ((h - 1) >> 1) & 1, abort, args.status))) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int ch = 0; ch < 4; ++ch) {
              uint32_t oo[32];
              tmem_ld32(o_tmem + ch * 32, oo);
              tmem_ld_wait();
#pragma unroll
              for (int x = 0; x < 32; ++x) oo[x] = __float_as_uint(__uint_as_float(oo[x]) * alpha);
              tmem_st32(o_tmem + ch * 32, oo);
            }
          }
          m_ref = m_new;
        }
        // p = exp2(s c - m_ref), written over S as the A operand of P V
        const float m_use = (m_ref == ninf) ? 0.f : m_ref;
        const float2 c2 = make_float2(c, c), nm2 = make_float2(-m_use, -m_use);
        float2 ps0 = make_float2(0.f, 0.f), ps1 = make_float2(0.f, 0.f);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          uint32_t w[16];
          if constexpr (kPolyMask == 0u) {
            exp_chunk<0u, kFp8>(rr[ch], c2, nm2, ps0, ps1, w);  // one copy of the code for every half
          } else if (diag) {
            exp_chunk<0u, kFp8>(rr[ch], c2, nm2, ps0, ps1, w);  // masked keys need an exact 0
          } else {
            exp_chunk<kPolyMask, kFp8>(rr[ch], c2, nm2, ps0, ps1, w);
          }
          tmem_st16(s_tmem + 16 * ch, w);  // 32 keys -> 16 columns at 16 ch
        }
        l += (ps0.x + ps0.y) + (ps1.x + ps1.y);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[t][half]);
      }
    }

    // epilogue: normalise O and store this row (the TMEM reads are warp-wide;
    // only rows inside the sequence are stored)
    {
      const bool have_o = ok && N > 0 && __all_sync(0xffffffffu, mbar_wait(&sm.o_done[t], 0, abort, args.status));
      if (have_o) tc_fence_after();
      const bool store = t_row < L;
      float inv = (l > 0.f) ? 1.f / l : 0.f;
      if constexpr (kFp8) inv *= args.v_scale[tl.hk];
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint8_t*>(args.out) +
                                            (tok * args.hq + tl.h) * static_cast<size_t>(kHeadDim) * 2);
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t rr[32];
        if (have_o) {
          tmem_ld32(o_tmem + ch * 32, rr);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) rr[x] = 0u;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = pack_bf16x2(__uint_as_float(rr[q * 8 + 2 * e]) * inv, __uint_as_float(rr[q * 8 + 2 * e + 1]) * inv);
          if (store) dst[ch * 4 + q] = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      const float lse = (l > 0.f) ? (m_ref + __log2f(l)) * 0.69314718055994530942f : ninf;
      if (store) args.lse[static_cast<size_t>(tl.h) * args.total_tokens + tok] = lse;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kPairMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kPairTmemCols);
  }
}

// Above half of the SM's shared memory, so that one CTA (which allocates all
// of the SM's tensor memory) runs per SM.
size_t bsa_pair_smem_bytes(bool fp8) {
  const size_t need = (fp8 ? sizeof(PairSmem<true>) : sizeof(PairSmem<false>)) + 1024;
  return need > (size_t(116) << 10) ? need : (size_t(116) << 10);
}

cudaError_t launch_bsa_pair(const BsaMaps& maps, const SeqBatch& batch, const BsaArgs& args, bool fp8,
                            cudaStream_t stream) {
  const int items = batch.item0[batch.n];
  if (items == 0) return cudaSuccess;
  const size_t smem = bsa_pair_smem_bytes(fp8);
  cudaError_t e;
  if (fp8) {
    e = cudaFuncSetAttribute(bsa_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bsa_pair_kernel<true><<<items, kPairThreads, smem, stream>>>(maps, batch, args);
  } else {
    e = cudaFuncSetAttribute(bsa_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    bsa_pair_kernel<false><<<items, kPairThreads, smem, stream>>>(maps, batch, args);
  }
  return cudaGetLastError();
}

}  // namespace stem
