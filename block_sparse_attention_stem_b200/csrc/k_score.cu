// k_score.cu — block scores of the output-aware metric on the tensor cores.
//
// AngelSlim documentation §2.1 (score = Q.K^T / (sqrt(d) s n) from a strided
// group GEMM), "Stem" gist.science zh §2.3 / de §2 C (anti-diagonal
// downsampling), zh §2.2 (M_ij = routing score + beta max(0, log||V_j||^2)).
//
//   D[a][b] = sum_{u<s} q[a s + u] . k[b s + s-1-u] / (sqrt(d) s n)
//   S[i][j] = max_{a in block i, b in block j} D[a][b] + vbonus[j]
//
// D is a plain GEMM with reduction length s*d: query group a contributes the
// s token rows a s + u (slot u), key group b the rows b s + s-1-u.  Each CTA
// owns one (sequence, pair of query heads of one KV group, 128-group query
// tile I) and walks the 256-group key tiles J that reach its causal range.
// Slot tiles are fetched by TMA with a token traversal stride of s (one tensor
// map per sequence, so rows past the sequence end arrive as zeros), staged
// 128-B swizzled, and fed to tcgen05.mma (M = 128, N = 256, fp32 in TMEM, one
// 256-column accumulator per head).  The two heads share every staged key
// tile: a 64 KB stage (two 16 KB query slabs, one 32 KB key slab) feeds 1024
// tensor cycles, where a single head's 48 KB stage fed 512.  The bytes moved
// from L2 into shared memory per product are what bound this GEMM, so sharing
// the key slab is what pays.  The epilogue warps (two warpgroups per head, one
// per half of the accumulator's columns) read their TMEM lane quarter,
// max-pool 16 columns in registers and 16 rows with
// warp shuffles, scale, add the bonus and write one fp32 score per (query
// block, key block); the next tile's products on a head wait only for that
// head's epilogue.
//
// Warp roles (576 threads): epilogue warps 0-15, warp w on head (w / 4) % 2,
// TMEM lane quarter w % 4 and TMEM columns 128 (w / 8) .. +127 (two warps per
// lane quarter, so a tile's accumulator is read back in half the time), warp
// 16 TMA producer, warp 17 TMEM owner + MMA issuer.
#include "stem_device.cuh"
#include "stem_kernels.h"
#include "stem_select_row.cuh"

namespace stem {

namespace {

constexpr int kScoreThreads = 576;
constexpr int kProducerWarp = 16;
constexpr int kMmaWarp = 17;
constexpr int kTileM = 128;            // query groups per tile (MMA M)
constexpr int kTileN = 256;            // key groups per tile (MMA N)
constexpr int kBytesA = kTileM * 128;  // one 128-B row per group and K-chunk, per head
constexpr int kBytesB = kTileN * 128;
constexpr int kStageBytes = 2 * kBytesA + kBytesB;  // 64 KB: A of both heads, then B
constexpr int kScoreStages = 3;
constexpr uint32_t kScoreTmemCols = 512;  // head e: 256-column accumulator at 256 e

struct ScoreSmem {
  uint8_t stage[kScoreStages][kStageBytes];  // 1024-aligned (swizzle atoms)
  uint64_t full[kScoreStages];
  uint64_t empty[kScoreStages];
  uint64_t acc_full;      // the products of tile J are complete (both heads)
  uint64_t acc_empty[2];  // per head: its epilogue read tile J
  uint64_t drain;         // completion of every MMA this CTA issued
  uint32_t tmem_base;
  int abort;
};

}  // namespace

template <bool kFp8, int kS, int kB>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ ScoreMaps maps, const SeqBatch batch, const ScoreArgs args) {
  extern __shared__ uint8_t smem_raw[];
  ScoreSmem& sm = *reinterpret_cast<ScoreSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = warp_id(), lane = lane_id();
  const int seq = find_seq(batch, blockIdx.x);
  const int local = blockIdx.x - batch.item0[seq];
  constexpr int s = kS;  // scoring stride (compile-time so the pooling indices are)
  constexpr int gpb = kB / s;                      // groups per block (16 for 128-token blocks, s = 8)
  constexpr int kBlocksPerTile = kTileM / gpb;     // query blocks per 128-group query tile
  const int nb = batch.nb[seq];
  const int L = batch.len[seq];
  const int ntile = (nb + kBlocksPerTile - 1) / kBlocksPerTile;
  // KV heads in groups of g; inside a group, query tiles descending (query
  // tile, KV head, head pair of the group).  A CTA's work grows with its
  // query tile.  When one KV head's CTAs outnumber the SMs, g = 1: the CTAs in
  // flight stream one KV head's keys, which stay in L2, and the tail is short
  // anyway.  Otherwise one KV head would leave the SMs unevenly loaded, and g
  // is the largest divisor of the launch's KV heads whose keys fit in 64 MB,
  // so each group starts its longest CTAs first and short ones fill the tail.
  const int G = args.hq / args.hkv;
  const int npair = (G + 1) / 2;
  const int nhk = (batch.item0[seq + 1] - batch.item0[seq]) / (npair * ntile);  // KV heads in this launch
  int g = 1;
  if (npair * ntile < args.num_sms) {
    const size_t key_bytes = static_cast<size_t>(L) * 128 * (kFp8 ? 1 : 2);  // one KV head's keys
    for (int c = nhk; c > 1; --c)
      if (nhk % c == 0 && static_cast<size_t>(c) * key_bytes <= (size_t(64) << 20)) {
        g = c;
        break;
      }
  }
  const int lg = local % (g * npair * ntile);
  const int I = ntile - 1 - lg / (g * npair);
  const int rem = lg % (g * npair);
  const int hk = args.hk0 + (local / (g * npair * ntile)) * g + rem / npair;
  const int h0 = hk * G + 2 * (rem % npair);
  const bool has1 = 2 * (rem % npair) + 1 < G;  // an odd group leaves the last pair one head
  const int halves = kFp8 ? 1 : 2;       // 64-element (bf16) or 128-element (fp8) K chunks per slot
  const int stages_per_tile = s * halves;
  const int rows_per_load = 256 / s;     // TMA box of 256 tokens traversed with stride s
  const int loads_a = kTileM / rows_per_load;
  const int loads_b = kTileN / rows_per_load;
  const int load_bytes = rows_per_load * 128;
  const int jmax = (I * kTileM + kTileM - 1) / kTileN;  // last key tile reaching the query tile

  if (threadIdx.x == 0) {
    for (int i = 0; i < kScoreStages; ++i) {
      mbar_init(&sm.full[i], 1);
      mbar_init(&sm.empty[i], 1);
    }
    mbar_init(&sm.acc_full, 1);
    for (int i = 0; i < 2; ++i) mbar_init(&sm.acc_empty[i], 8);
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, kScoreTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      const CUtensorMap* mq = &maps.q[seq];
      const CUtensorMap* mk = &maps.k[seq];
      tma_prefetch_desc(mq);
      tma_prefetch_desc(mk);
      const bool grouped = maps.group_maps[seq] != 0;
      const CUtensorMap* mqg = &maps.q_groups[seq];
      const CUtensorMap* mkg = &maps.k_groups[seq];
      if (grouped) {
        tma_prefetch_desc(mqg);
        tma_prefetch_desc(mkg);
      }
      // the partial last group (L % s tokens) lies outside the group maps
      const int gpart = (L % s != 0) ? L / s : -1;
      auto holds_partial = [&](int g0, int n) { return gpart >= g0 && gpart < g0 + n; };
      const bool a_grouped = grouped && !holds_partial(I * kTileM, kTileM);
      int stage = 0;
      uint32_t phase = 0;
      int filled = 0;
      bool ok = true;
      for (int J = 0; J <= jmax && ok; ++J) {
        for (int t = 0; t < stages_per_tile && ok; ++t) {
          const int u = t / halves, hh = t % halves;
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort, args.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.full[stage], (has1 ? 2 : 1) * kBytesA + kBytesB);
          uint8_t* sa = sm.stage[stage];
          uint8_t* sb = sm.stage[stage] + 2 * kBytesA;
          const int ta = (I * kTileM) * s + u;
          const int tb = (J * kTileN) * s + (s - 1 - u);
          // whole-group tiles: one copy per operand slab; the tile holding a
          // partial last group: s-strided copies of 32 rows (zeros past the end)
          if (a_grouped) {
            for (int e = 0; e < (has1 ? 2 : 1); ++e)
              tma_load_4d(sa + e * kBytesA, mqg, &sm.full[stage], hh * 64, h0 + e, u, I * kTileM);
          } else {
            for (int e = 0; e < (has1 ? 2 : 1); ++e)
              for (int c = 0; c < loads_a; ++c)
                tma_load_3d(sa + e * kBytesA + c * load_bytes, mq, &sm.full[stage], hh * 64, h0 + e,
                            ta + c * rows_per_load * s);
          }
          if (grouped && !holds_partial(J * kTileN, kTileN)) {
            tma_load_4d(sb, mkg, &sm.full[stage], hh * 64, hk, s - 1 - u, J * kTileN);
          } else {
            for (int c = 0; c < loads_b; ++c)
              tma_load_3d(sb + c * load_bytes, mk, &sm.full[stage], hh * 64, hk, tb + c * rows_per_load * s);
          }
          ++filled;
          if (++stage == kScoreStages) { stage = 0; phase ^= 1u; }
        }
      }
      // every copy has landed before the CTA can exit (a stage holds at most
      // one round in flight: the next round into it waits for its consumer)
      for (int x = 0; x < kScoreStages && x < filled; ++x) {
        const int last = filled - 1 - ((filled - 1 - x) % kScoreStages);  // last fill of stage x
        mbar_wait_quiesce(&sm.full[x], (last / kScoreStages) & 1, args.status);
      }
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(kFp8 ? 0u : 1u, 0u, 128u, 256u);
      const int nh = has1 ? 2 : 1;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int J = 0; J <= jmax && ok; ++J) {
        for (int t = 0; t < stages_per_tile; ++t) {
          if (!mbar_wait(&sm.full[stage], phase, abort, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm.stage[stage]);
          const uint32_t sb = sa + 2 * kBytesA;
          for (int e = 0; e < nh && ok; ++e) {
            // a head's accumulator is overwritten from its first product of
            // tile J on: its epilogue must have read tile J-1
            if (t == 0) {
              ok = mbar_wait(&sm.acc_empty[e], (J & 1) ^ 1u, abort, args.status);
              if (!ok) break;
              tc_fence_after();
            }
            const uint32_t d_tmem = tmem + 256 * e;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint64_t ad = make_sdesc_sw128(sa + e * kBytesA + kk * 32, 16, 1024);
              const uint64_t bd = make_sdesc_sw128(sb + kk * 32, 16, 1024);
              if constexpr (kFp8) mma_f8_ss(d_tmem, ad, bd, idesc, (t | kk) != 0);
              else mma_bf16_ss(d_tmem, ad, bd, idesc, (t | kk) != 0);
            }
          }
          if (!ok) break;
          mma_commit(&sm.empty[stage]);
          if (++stage == kScoreStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) mma_commit(&sm.acc_full);
      }
      // no MMA may still run when TMEM is released
      mma_commit(&sm.drain);
      mbar_wait_quiesce(&sm.drain, 0, args.status);
    }
    __syncwarp();
  } else if (((warp >> 2) & 1) == 0 || has1) {
    // epilogue: warpgroups e and e + 2 handle head h0 + e, the first the key
    // groups of TMEM columns 0-127 of each tile, the second columns 128-255;
    // thread owns TMEM lane (query group of the tile) `row`
    const int e = (warp >> 2) & 1;
    const int half = warp >> 3;
    const int h = h0 + e;
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const int a = I * kTileM + row;              // query group within the sequence
    const bool row_valid = a * s < L;
    const int i = a / gpb;                       // query block (local)
    const int g = batch.g0[seq] + i;
    float scale = args.scale;
    if constexpr (kFp8) scale *= args.q_scale[h] * args.k_scale[hk];
    const float* bonus = args.vbonus + static_cast<size_t>(hk) * args.nbtot + batch.g0[seq];
    float* srow = args.scores + (static_cast<size_t>(h) * args.nbtot + g) * args.nb_max;
    const bool writer = (lane % gpb) == 0 && row_valid && i < nb;
    const float ninf = -__int_as_float(0x7f800000);
    constexpr int kbt = kTileN / gpb;    // key blocks per key tile (at most 32: one per lane)
    constexpr int kbc = 32 / gpb;        // key blocks per 32-column chunk
    constexpr int kbh = kbt / 2;         // key blocks per half tile
    bool complete = true;
    for (int J = 0; J <= jmax; ++J) {
      // every lane waits; the warp leaves together if any lane gave up
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full, J & 1, abort, args.status))) {
        complete = false;
        break;
      }
      tc_fence_after();
      // 1. pool each key block's gpb key groups in registers, straight out of
      //    TMEM (groups past the end of the sequence excluded) ...
      float pooled[kbh];
#pragma unroll
      for (int ch = 0; ch < 4; ch += 2) {
        uint32_t r[2][32];  // two 32-column chunks per TMEM wait
        const uint32_t col = e * 256 + half * 128 + ch * 32;
        tmem_ld32(tmem + col + (static_cast<uint32_t>(q4 * 32) << 16), r[0]);
        tmem_ld32(tmem + col + 32 + (static_cast<uint32_t>(q4 * 32) << 16), r[1]);
        tmem_ld_wait();
#pragma unroll
        for (int c2 = 0; c2 < 2; ++c2) {
          const int b0 = J * kTileN + half * 128 + (ch + c2) * 32;  // first key group of the chunk
          const bool inside = (b0 + 32) * s <= L;      // no group of the chunk past the end
#pragma unroll
          for (int kb = 0; kb < kbc; ++kb) {
            const int c0 = kb * gpb;
            float v = ninf;
            if (inside) {
#pragma unroll
              for (int cc = c0; cc < c0 + gpb; cc += 2)
                v = fmax3(v, __uint_as_float(r[c2][cc]), __uint_as_float(r[c2][cc + 1]));
            } else {
#pragma unroll
              for (int cc = c0; cc < c0 + gpb; cc += 2)
                v = fmax3(v, ((b0 + cc) * s < L) ? __uint_as_float(r[c2][cc]) : ninf,
                          ((b0 + cc + 1) * s < L) ? __uint_as_float(r[c2][cc + 1]) : ninf);
            }
            pooled[(ch + c2) * kbc + kb] = v;
          }
        }
      }
      // ... then hand the accumulator back: the next tile's products on this
      // head can start while the rest of the epilogue runs
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[e]);
      // 2. the max over the gpb query groups (consecutive lanes) of each query
      //    block, scale, bonus (lane k holds the tile's k-th key block's), store
      const int jl = J * kbt + lane;
      const float bl = (lane < kbt && jl < nb) ? bonus[jl] : 0.f;
#pragma unroll
      for (int k = 0; k < kbh; ++k) {  // unrolled, so that pooled[] stays in registers
        float v = row_valid ? pooled[k] : ninf;
#pragma unroll
        for (int off = gpb / 2; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
        const float bk = __shfl_sync(0xffffffffu, bl, half * kbh + k);
        const int j = J * kbt + half * kbh + k;
        if (writer && j < args.nb_max) srow[j] = (j <= i) ? fmaf(v, scale, 0.f) + bk : ninf;
      }
      if (J == jmax && writer && half == 0)
        for (int j = (jmax + 1) * kbt; j < args.nb_max; ++j) srow[j] = ninf;
    }
    // the two warps of a lane quarter wrote the two halves of the same rows:
    // both reach this barrier once, whatever ended their loop
    switch (e * 4 + q4) {  // constant barrier ids 1-8, one per (head, lane quarter)
      case 0: asm volatile("bar.sync 1, 64;" ::: "memory"); break;
      case 1: asm volatile("bar.sync 2, 64;" ::: "memory"); break;
      case 2: asm volatile("bar.sync 3, 64;" ::: "memory"); break;
      case 3: asm volatile("bar.sync 4, 64;" ::: "memory"); break;
      case 4: asm volatile("bar.sync 5, 64;" ::: "memory"); break;
      case 5: asm volatile("bar.sync 6, 64;" ::: "memory"); break;
      case 6: asm volatile("bar.sync 7, 64;" ::: "memory"); break;
      default: asm volatile("bar.sync 8, 64;" ::: "memory"); break;
    }
    if (args.fuse_select && complete && half == 0) {
      // Select the rows this lane quarter scored: the query blocks whose
      // groups are its 32 lanes (their scores were written by the writer
      // lanes of this warp and of its partner for the upper half of each tile;
      // the barrier above orders those stores for both).  Every product of
      // the CTA has completed (the last acc_full), so the operand stages are
      // free: they hold each selecting warp's keys and histogram.
      __syncwarp();
      const size_t key_bytes = (static_cast<size_t>(args.nb_max) * 4 + 15) & ~size_t(15);
      uint8_t* scratch = sm.stage[0] + static_cast<size_t>(warp) * (key_bytes + 1024);
      uint32_t* keys = reinterpret_cast<uint32_t*>(scratch);
      int* hist = reinterpret_cast<int*>(scratch + key_bytes);
      for (int rb = 0; rb < 32 / gpb; ++rb) {
        const int ib = (I * kTileM + q4 * 32) / gpb + rb;  // query block (local)
        if (ib >= nb) break;
        const size_t r = static_cast<size_t>(h) * args.nbtot + batch.g0[seq] + ib;
        warp_select_row(args.scores + r * static_cast<size_t>(args.nb_max), ib, args.budgets[r], args.sink,
                        args.window, keys, hist, args.col_idx, args.row_ptr, r);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kScoreTmemCols);
  }
}

size_t score_smem_bytes() { return sizeof(ScoreSmem) + 1024; }

template <bool kFp8, int kS, int kB>
static cudaError_t launch_score_t(const ScoreMaps& maps, const SeqBatch& batch, const ScoreArgs& args,
                                  cudaStream_t stream) {
  const size_t smem = score_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(score_kernel<kFp8, kS, kB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  score_kernel<kFp8, kS, kB><<<batch.item0[batch.n], kScoreThreads, smem, stream>>>(maps, batch, args);
  return cudaGetLastError();
}

template <int kS, int kB>
static cudaError_t launch_score_b(const ScoreMaps& maps, const SeqBatch& batch, const ScoreArgs& args, bool fp8,
                                  cudaStream_t stream) {
  return fp8 ? launch_score_t<true, kS, kB>(maps, batch, args, stream)
             : launch_score_t<false, kS, kB>(maps, batch, args, stream);
}

cudaError_t launch_score(const ScoreMaps& maps, const SeqBatch& batch, const ScoreArgs& args_in, bool fp8,
                         cudaStream_t stream) {
  if (batch.item0[batch.n] == 0) return cudaSuccess;
  ScoreArgs args = args_in;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&args.num_sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const bool b64 = args.block == kBlock / 2;
  if (!b64 && args.block != kBlock) return cudaErrorInvalidValue;
  if (args.stride == 8)
    return b64 ? launch_score_b<8, 64>(maps, batch, args, fp8, stream) : launch_score_b<8, 128>(maps, batch, args, fp8, stream);
  if (args.stride == 4)
    return b64 ? launch_score_b<4, 64>(maps, batch, args, fp8, stream) : launch_score_b<4, 128>(maps, batch, args, fp8, stream);
  return cudaErrorInvalidValue;
}

}  // namespace stem
