// k_bsa.cu — causal block-sparse flash attention over pre-compacted block lists.
//
// "Stem" gist.science zh §2.3 (exact softmax and aggregation only over the
// selected blocks); youleyou HPC-BSA article §3.1 (the inner loop walks a list
// prepared outside it; a skipped block is the same as a block of -inf scores,
// so the softmax needs no change; fixed 128 x 128 tiles).
//
// One CTA owns one CSR row (a query block i of one query head); two CTAs run
// on every SM, each with half of the SM's tensor memory, so the two rows
// proceed independently and one CTA's start-up and epilogue overlap the other
// CTA's main loop.  Rows are taken in KV-head-major, longest-first order, so
// the CTAs in flight share one KV head's K/V in L2.  Every listed key block j
// (ascending, the diagonal last) is processed as two halves of 64 keys,
// h = 2n and 2n + 1:
//   S_h = Q K_h^T          tcgen05.mma (M 128, N 64), Q and K from SMEM, fp32
//                          into S buffer h % 2 (TMEM)
//   P_h = exp2(S_h c - m)  the softmax warpgroup (thread = query row = TMEM
//                          lane); P is written back over S_h
//   O += P_h V_h           tcgen05.mma with P from TMEM, V from SMEM
//                          (MN-major); the fp32 accumulator stays in TMEM
// With two S buffers, S_{h+1} is computed while the softmax of half h runs, so
// the softmax does not wait for the tensor core in steady state.
// The reference row max m moves (and O is rescaled in TMEM) only when a half
// raises it past a threshold (2^8), so P stays bounded and
// rescales are rare; O and the row sum share that reference, so the result is
// exact.  A rescale first waits for P_{h-1} V_{h-1} (S_h does not imply it).
// Masking happens only on the diagonal block.
//
// fp8: Q K^T runs on e4m3 operands (kind::f8f6f4).  A single e4m3 P would
// carry three mantissa bits (up to 6% error per weight, which rows with few
// keys cannot average out), so P is kept in f16 and P V runs as an f16
// product (kind::f16) against V widened to f16 beforehand (every e4m3 value is
// an f16 value, so the widening is exact).  Two e4m3 products of a split P
// would take the same tensor time as the one f16 product, and more
// conversions per weight.
//
// P is written over S in place: chunk ch (keys 32ch..32ch+31 of the half)
// goes to columns 16ch..16ch+15 of the S buffer (bf16 or f16 pairs); the whole
// half is in registers by then.
//
// Warp roles (224 threads):
//   warps 0-3  softmax + epilogue (TMEM lane quarters 0-3)
//   warp  4    TMA producer of Q and the K halves (and stages the block list)
//   warp  5    TMA producer of the V halves (one issuing thread moves only
//              about 26 B per cycle, so K and V get a thread each)
//   warp  6    TMEM owner and MMA issuer
// Half h uses K slot and V slot h % 2: K_{h+2} may overwrite K_h once S_h is
// complete, V_{h+2} may overwrite V_h once P_h V_h is, so a product needs one
// commit.  Block lists are staged in shared memory; every wait is bounded.
//
// 64-token blocks (the "64x128" KV blocks of the HPC-BSA article §3.1): a
// tcgen05.mma with M = 64 takes as long as one with M = 128, so the CTA keeps
// its 128-row tile and gives it query blocks 2p and 2p + 1 (rows 0-63 and
// 64-127).  Their two lists are staged as bitmaps of key blocks, and the CTA
// walks the union in ascending order, one 64-key unit per listed block, with
// the same S / P / P V pipeline as the halves above.  A unit in only one of
// the lists is a block of -inf scores for the other block's rows: those warps
// store P = 0 and skip the exponentials.
#include "stem_bsa_common.cuh"

namespace stem {

namespace {

constexpr int kBsaThreads = 224;
constexpr int kKProducerWarp = 4;
constexpr int kVProducerWarp = 5;
constexpr int kMmaWarp = 6;
constexpr uint32_t kBsaTmemCols = 256;  // S buffers at 0 and 64, O at 128

template <bool kFp8>
struct BsaSmem {
  uint8_t q[BsaCfg<kFp8>::kQBytes];                        // 1024-aligned
  uint8_t k[2][BsaCfg<kFp8>::kKHalfBytes];                 // per slot
  uint8_t v[2][BsaCfg<kFp8>::kVHalfBytes];
  uint64_t q_full;
  uint64_t k_full[2];  // per slot: K_h landed
  uint64_t v_full[2];  // per slot: V_h landed
  uint64_t s_full[2];  // per S buffer: S_h complete (K slot free again)
  uint64_t v_free[2];  // per slot: P_h V_h complete (V slot free again)
  uint64_t p_full[2];  // per S buffer: the 4 softmax warps stored P_h (and rescaled O)
  uint64_t o_done;     // the last P V is complete
  uint64_t drain;      // every MMA of the issuer complete
  int32_t list[kMaxList];
  int nvalid;
  int in_smem;
  uint32_t tmem_base;
  int abort;
};

// 64-token blocks: the lists of query blocks 2p and 2p + 1 (rows 0-63 and
// 64-127 of the CTA's 128-token tile) as two bitmaps of key blocks in the
// list storage (words 0 .. 1023 and 1024 .. 2047); *nunits = size of their
// union.  Valid entries as for the staged list (0 <= j <= the row's block,
// above the previous valid entry); a malformed list is compacted entry by
// entry and reported.  One whole warp.
constexpr int kBitmapWords = kMaxBitmapBlocks / 32;
static_assert(2 * kBitmapWords <= kMaxList, "two bitmaps must fit the list storage");

__device__ void stage_bitmaps(const int32_t* __restrict__ col, int beg0, int end0, int i0, int beg1, int end1,
                              int i1, int nwords, uint32_t* bm, int* nunits, int* status) {
  const int lane = lane_id();
  for (int w = lane; w < nwords; w += 32) {
    bm[w] = 0u;
    bm[kBitmapWords + w] = 0u;
  }
  __syncwarp();
  for (int e = 0; e < 2; ++e) {
    const int beg = e ? beg1 : beg0, end = e ? end1 : end0, i = e ? i1 : i0;
    uint32_t* b = bm + e * kBitmapWords;
    bool good = true;
    for (int p0 = beg; p0 < end; p0 += 32) {
      const int p = p0 + lane;
      const int j = p < end ? __ldg(col + p) : 0;
      int before = __shfl_up_sync(0xffffffffu, j, 1);
      if (lane == 0) before = p0 > beg ? __ldg(col + p0 - 1) : -1;
      if (__any_sync(0xffffffffu, p < end && (j < 0 || j > i || j <= before))) {
        good = false;
        break;
      }
      if (p < end) atomicOr(b + (j >> 5), 1u << (j & 31));
    }
    __syncwarp();
    if (!good && lane == 0) {
      set_status(status, STEM_ERR_BAD_BLOCKLIST_CODE);
      for (int w = 0; w < nwords; ++w) b[w] = 0u;
      int prev = -1, j = 0;
      for (int p = next_valid(col, beg, end, prev, i, &j); p < end; p = next_valid(col, p + 1, end, prev, i, &j)) {
        b[j >> 5] |= 1u << (j & 31);
        prev = j;
      }
    }
    __syncwarp();
  }
  int n = 0;
  for (int w = lane; w < nwords; w += 32) n += __popc(bm[w] | bm[kBitmapWords + w]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
  if (lane == 0) *nunits = n;
}

// Walks the union of the two bitmaps in ascending key-block order.
struct BitmapCursor {
  int w = -1;
  uint32_t bits = 0u;
  __device__ __forceinline__ int next(const uint32_t* bm) {
    while (bits == 0u && w + 1 < kBitmapWords) {
      ++w;
      bits = bm[w] | bm[kBitmapWords + w];
    }
    const int b = __ffs(bits) - 1;
    bits &= bits - 1u;
    return w * 32 + b;
  }
};

}  // namespace

template <bool kFp8, bool kB64>
__global__ void __launch_bounds__(kBsaThreads, 2)
    bsa_kernel(const __grid_constant__ BsaMaps maps, const SeqBatch batch, const BsaArgs args) {
  using Cfg = BsaCfg<kFp8>;
  extern __shared__ uint8_t smem_raw[];
  BsaSmem<kFp8>& sm =
      *reinterpret_cast<BsaSmem<kFp8>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = warp_id(), lane = lane_id();
  const int seq = find_seq(batch, blockIdx.x);
  const int nb = batch.nb[seq];
  const int L = batch.len[seq];
  const int G = args.hq / args.hkv;
  // Rows of a sequence in KV-head-major order: KV head, then query blocks
  // descending (longest rows first), then the query heads of the group.
  // tl.i: the 128-token query tile (query block i, or with 64-token blocks
  // query blocks 2i and 2i + 1, whose second CSR range is beg1 .. end1)
  const int ntiles = kB64 ? (nb + 1) / 2 : nb;
  Tile tl;
  int beg1 = 0, end1 = 0;
  {
    const int it = blockIdx.x - batch.item0[seq];
    const int hk_of = args.hk0 + it / (G * ntiles);
    const int rem = it % (G * ntiles);
    tl.valid = true;
    tl.i = ntiles - 1 - rem / G;
    tl.h = hk_of * G + rem % G;
    tl.hk = tl.h / G;
    const size_t r = static_cast<size_t>(tl.h) * args.nbtot + batch.g0[seq] + (kB64 ? 2 * tl.i : tl.i);
    tl.beg = args.row_ptr[r];
    tl.end = args.row_ptr[r + 1];
    if (kB64 && 2 * tl.i + 1 < nb) {
      beg1 = args.row_ptr[r + 1];
      end1 = args.row_ptr[r + 2];
    }
  }
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(sm.list);

  if (warp == kKProducerWarp) {
    if constexpr (kB64) {
      stage_bitmaps(args.col_idx, tl.beg, tl.end, 2 * tl.i, beg1, end1, 2 * tl.i + 1, (nb + 31) / 32, bitmaps,
                    &sm.nvalid, args.status);
      if (lane_id() == 0) sm.in_smem = 1;
    } else {
      stage_list(args.col_idx, tl, sm.list, &sm.nvalid, &sm.in_smem, args.status);
    }
  }
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.k_full[b], 1);
      mbar_init(&sm.v_full[b], 1);
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.v_free[b], 1);
      mbar_init(&sm.p_full[b], 4);
    }
    mbar_init(&sm.o_done, 1);
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
  const int N = sm.nvalid;
  const bool list_in_smem = sm.in_smem != 0;
  volatile int* abort = &sm.abort;

  if (warp == kKProducerWarp || warp == kVProducerWarp) {
    // ------------------------------------------------------------ producers
    const bool is_v = warp == kVProducerWarp;
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
        mbar_arrive_expect_tx(&sm.q_full, Cfg::kQBytes);
        for (int hh = 0; hh < Cfg::kKSlabs; ++hh)
          tma_load_3d(sm.q + hh * 16384, &maps.q[seq], &sm.q_full, hh * 64, tl.h, tl.i * kBlock);
      }
      const int H = kB64 ? N : 2 * N;  // 64-key units
      ListCursor cur(tl.beg);
      BitmapCursor bcur;
      int j = 0, issued = 0;
      for (int h = 0; h < H; ++h) {
        if (h >= 2) {
          uint64_t* freed = is_v ? &sm.v_free[h & 1] : &sm.s_full[h & 1];
          if (!mbar_wait(freed, ((h - 2) >> 1) & 1, abort, args.status)) break;
        }
        if (kB64) j = bcur.next(bitmaps);
        else if ((h & 1) == 0) j = cur.next(sm.list, list_in_smem, h >> 1, args.col_idx, tl.end, tl.i);
        uint8_t* dst = is_v ? sm.v[h & 1] : sm.k[h & 1];
        uint64_t* bar = is_v ? &sm.v_full[h & 1] : &sm.k_full[h & 1];
        // token row of the unit: in the sequence, or through the page table (a
        // 64-key unit never straddles a page; a page number outside the pool
        // reads zeros)
        int row = kB64 ? j * kHalf : j * kBlock + (h & 1) * kHalf;
        if (paged) row = __ldg(pages + row / args.page_size) * args.page_size + row % args.page_size;
        mbar_arrive_expect_tx(bar, half_bytes);
        for (int hh = 0; hh < slabs; ++hh) tma_load_3d(dst + hh * (kHalf * 128), m, bar, hh * 64, tl.hk, row);
        ++issued;
      }
      // every copy of this producer has landed before the CTA can exit (a
      // slot holds at most one copy in flight: the next copy into it waits
      // for the product that consumes this one)
      if (!is_v) mbar_wait_quiesce(&sm.q_full, 0, args.status);
      for (int x = 0; x < 2 && x < issued; ++x) {
        const int last = issued - 1 - ((issued - 1 - x) & 1);  // last half issued into slot x
        mbar_wait_quiesce(is_v ? &sm.v_full[x] : &sm.k_full[x], (last >> 1) & 1, args.status);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && N > 0) {
      const uint32_t idesc_s = make_idesc(kFp8 ? 0u : 1u, 0u, 128u, static_cast<uint32_t>(kHalf));
      const uint32_t idesc_o = make_idesc(kFp8 ? 0u : 1u, 1u, 128u, 128u);  // kind::f16: f16 (0) or bf16 (1)
      const uint32_t sq = smem_u32(sm.q);
      const uint32_t o_tmem = tmem + 128;
      const int H = kB64 ? N : 2 * N;
      auto issue_s = [&](int h) -> bool {  // S_h = Q K_h^T into buffer h % 2
        if (!mbar_wait(&sm.k_full[h & 1], (h >> 1) & 1, abort, args.status)) return false;
        tc_fence_after();
        const uint32_t sk = smem_u32(sm.k[h & 1]);
        const uint32_t d = tmem + kHalf * (h & 1);
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
        mma_commit(&sm.s_full[h & 1]);
        return true;
      };
      auto issue_pv = [&](int h) -> bool {  // O += P_h V_h
        if (!mbar_wait(&sm.p_full[h & 1], (h >> 1) & 1, abort, args.status)) return false;
        if (!mbar_wait(&sm.v_full[h & 1], (h >> 1) & 1, abort, args.status)) return false;
        tc_fence_after();
        const uint32_t sv = smem_u32(sm.v[h & 1]);
        const uint32_t p = tmem + kHalf * (h & 1);
        // kind::f16 for both: bf16 P and V, or f16 P and V (the fp8 path)
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 keys per step
          mma_bf16_ts(o_tmem, p + kk * 8, make_sdesc_sw128(sv + kk * 2048, kHalf * 128, 1024), idesc_o,
                      (h | kk) != 0);
        mma_commit(&sm.v_free[h & 1]);
        if (h == H - 1) mma_commit(&sm.o_done);
        return true;
      };
      // S_0, S_1, then per half h: P_h V_h and S_{h+2} (into the buffer P_h
      // V_h just read: the tensor core runs one issuer's products in order)
      // (with 64-token blocks a tile may have a single unit)
      bool ok = mbar_wait(&sm.q_full, 0, abort, args.status) && issue_s(0) && (H < 2 || issue_s(1));
      for (int h = 0; h < H && ok; ++h) {
        ok = issue_pv(h);
        if (ok && h + 2 < H) ok = issue_s(h + 2);
      }
      // no MMA may still run when TMEM is released
      mma_commit(&sm.drain);
      mbar_wait_quiesce(&sm.drain, 0, args.status);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax + epilogue
    const int q4 = warp;  // TMEM lane quarter
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q4 * 32) << 16;
    const int t_row = tl.i * kBlock + row;  // token of this row inside the sequence
    const size_t tok = static_cast<size_t>(batch.tok0[seq]) + t_row;
    float c = args.scale_log2;  // sigma * log2(e) (* q_scale * k_scale for fp8)
    if constexpr (kFp8) c *= args.q_scale[tl.h] * args.k_scale[tl.hk];
    const float ninf = -__int_as_float(0x7f800000);
    const uint32_t s_base = tmem + lane_off;
    const uint32_t o_tmem = tmem + 128 + lane_off;

    float m_ref = ninf;  // reference max (scaled log2 domain) shared by O and l
    float l = 0.f;       // row sum of exp2(s c - m_ref)
    bool ok = true;
    ListCursor cur(tl.beg);
    BitmapCursor bcur;
    const int H = kB64 ? N : 2 * N;  // 64-key units
    int j = 0;
#pragma unroll 1
    for (int h = 0; h < H && ok; ++h) {
      {
        const int half = h & 1;  // S buffer of the unit
        // koff: the unit's first key minus the tile's first token (>= 0 only
        // on the diagonal, where keys above a row's token are masked)
        int koff;
        bool member = true;  // the unit is in the list of this warp's rows
        if constexpr (kB64) {
          j = bcur.next(bitmaps);
          koff = j * kHalf - tl.i * kBlock;
          member = ((bitmaps[(q4 >> 1) * kBitmapWords + (j >> 5)] >> (j & 31)) & 1u) != 0u;
        } else {
          if (half == 0) j = cur.next(sm.list, list_in_smem, h >> 1, args.col_idx, tl.end, tl.i);
          koff = (j == tl.i) ? half * kHalf : -kBlock;
        }
        const bool diag = koff >= 0;
        const uint32_t s_tmem = s_base + kHalf * half;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[half], (h >> 1) & 1, abort, args.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (kB64 && !member) {
          // the other query block's unit: P = 0 for these rows
          uint32_t z[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) z[x] = 0u;
          tmem_st16(s_tmem, z);
          tmem_st16(s_tmem + 16, z);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.p_full[half]);
          continue;
        }
        // the unit's 64 scores, loaded once and kept in registers
        uint32_t rr[2][32];
        tmem_ld32(s_tmem, rr[0]);
        tmem_ld32(s_tmem + 32, rr[1]);
        tmem_ld_wait();
        if (diag) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch)
#pragma unroll
            for (int x = 0; x < 32; ++x)
              if (koff + ch * 32 + x > row) rr[ch][x] = 0xff800000u;  // -inf -> p = 0
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
            // O holds P V up to unit h-1: let that product finish first
            if (!__all_sync(0xffffffffu,
                            mbar_wait(&sm.v_free[(h - 1) & 1], ((h - 1) >> 1) & 1, abort, args.status))) {
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
            exp_chunk<0u, kFp8>(rr[ch], c2, nm2, ps0, ps1, w);  // one copy of the code for every unit
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
        if (lane == 0) mbar_arrive(&sm.p_full[half]);
      }
    }

    // epilogue: normalise O and store this row (the TMEM reads are warp-wide;
    // only rows inside the sequence are stored)
    {
      const bool have_o = ok && N > 0 && __all_sync(0xffffffffu, mbar_wait(&sm.o_done, 0, abort, args.status));
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
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kBsaTmemCols);
  }
}

// At least 80 KB, so that no more than two CTAs share an SM's tensor memory
// (each allocates half of it; a third would wait in tcgen05.alloc).
size_t bsa_smem_bytes(bool fp8) {
  const size_t need = (fp8 ? sizeof(BsaSmem<true>) : sizeof(BsaSmem<false>)) + 1024;
  return need > (size_t(80) << 10) ? need : (size_t(80) << 10);
}

template <bool kFp8, bool kB64>
static cudaError_t launch_bsa_t(const BsaMaps& maps, const SeqBatch& batch, const BsaArgs& args, int items,
                                cudaStream_t stream) {
  const size_t smem = bsa_smem_bytes(kFp8);
  const cudaError_t e = cudaFuncSetAttribute(bsa_kernel<kFp8, kB64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  bsa_kernel<kFp8, kB64><<<items, kBsaThreads, smem, stream>>>(maps, batch, args);
  return cudaGetLastError();
}

cudaError_t launch_bsa(const BsaMaps& maps, const SeqBatch& batch, const BsaArgs& args, bool fp8,
                       cudaStream_t stream) {
  const int items = batch.item0[batch.n];
  if (items == 0) return cudaSuccess;
  if (args.block != kBlock && args.block != kHalf) return cudaErrorInvalidValue;
  const bool b64 = args.block == kHalf;
  return fp8 ? (b64 ? launch_bsa_t<true, true>(maps, batch, args, items, stream)
                    : launch_bsa_t<true, false>(maps, batch, args, items, stream))
             : (b64 ? launch_bsa_t<false, true>(maps, batch, args, items, stream)
                    : launch_bsa_t<false, false>(maps, batch, args, items, stream));
}

}  // namespace stem
