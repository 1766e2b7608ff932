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
// owns one (sequence, query head, 128-group query tile I) and walks the
// 256-group key tiles J that reach its causal range.  Slot tiles are fetched
// by TMA with a token traversal stride of s (one tensor map per sequence, so
// rows past the sequence end arrive as zeros), staged 128-B swizzled, and fed
// to tcgen05.mma (M = 128, N = 256, fp32 in TMEM, two accumulators so the
// epilogue of tile J overlaps the MMAs of J+1).  N = 256 makes every A read
// from shared memory serve twice as many products as N = 128, which is what
// bounds this GEMM (each operand byte is read from SMEM once per MMA).
// The epilogue warps read their TMEM lane quarter, max-pool 16 columns in
// registers and 16 rows with warp shuffles, scale, add the bonus and write one
// fp32 score per (query block, key block).
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 TMEM owner + MMA
// issuer, warps 2-5 epilogue (TMEM lane quarters 2, 3, 0, 1).
#include "stem_device.cuh"
#include "stem_kernels.h"

namespace stem {

namespace {

constexpr int kScoreThreads = 192;
constexpr int kTileM = 128;            // query groups per tile (MMA M)
constexpr int kTileN = 256;            // key groups per tile (MMA N)
constexpr int kBytesA = kTileM * 128;  // one 128-B row per group and K-chunk
constexpr int kBytesB = kTileN * 128;
constexpr int kStageBytes = kBytesA + kBytesB;  // 48 KB
constexpr int kScoreStages = 4;
constexpr uint32_t kScoreTmemCols = 512;  // two 256-column accumulators

struct ScoreSmem {
  uint8_t stage[kScoreStages][kStageBytes];  // 1024-aligned (swizzle atoms)
  uint64_t full[kScoreStages];
  uint64_t empty[kScoreStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;  // completion of every MMA this CTA issued
  uint32_t tmem_base;
  int abort;
};

}  // namespace

template <bool kFp8, int kS>
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ ScoreMaps maps, const SeqBatch batch, const ScoreArgs args) {
  extern __shared__ uint8_t smem_raw[];
  ScoreSmem& sm = *reinterpret_cast<ScoreSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int warp = warp_id(), lane = lane_id();
  const int seq = find_seq(batch, blockIdx.x);
  const int local = blockIdx.x - batch.item0[seq];
  constexpr int s = kS;  // scoring stride (compile-time so the pooling indices are)
  const int nb = batch.nb[seq];
  const int L = batch.len[seq];
  const int ntile = (nb + s - 1) / s;  // query tiles of 128 groups = s blocks
  // KV-head-major order (KV head, query tiles descending, heads of the group)
  // so the CTAs in flight share one KV head's keys in L2.
  const int G = args.hq / args.hkv;
  const int hk = local / (G * ntile);
  const int rem = local % (G * ntile);
  const int I = ntile - 1 - rem / G;  // longest rows first within a KV head
  const int h = hk * G + rem % G;
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
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.acc_full[i], 1);
      mbar_init(&sm.acc_empty[i], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kScoreTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap* mq = &maps.q[seq];
      const CUtensorMap* mk = &maps.k[seq];
      tma_prefetch_desc(mq);
      tma_prefetch_desc(mk);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int J = 0; J <= jmax && ok; ++J) {
        for (int t = 0; t < stages_per_tile && ok; ++t) {
          const int u = t / halves, hh = t % halves;
          if (!mbar_wait(&sm.empty[stage], phase ^ 1u, abort, args.status)) { ok = false; break; }
          mbar_arrive_expect_tx(&sm.full[stage], kStageBytes);
          uint8_t* sa = sm.stage[stage];
          uint8_t* sb = sm.stage[stage] + kBytesA;
          const int ta = (I * kTileM) * s + u;
          const int tb = (J * kTileN) * s + (s - 1 - u);
          for (int c = 0; c < loads_a; ++c)
            tma_load_3d(sa + c * load_bytes, mq, &sm.full[stage], hh * 64, h, ta + c * rows_per_load * s);
          for (int c = 0; c < loads_b; ++c)
            tma_load_3d(sb + c * load_bytes, mk, &sm.full[stage], hh * 64, hk, tb + c * rows_per_load * s);
          if (++stage == kScoreStages) { stage = 0; phase ^= 1u; }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc(kFp8 ? 0u : 1u, 0u, 128u, 256u);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int J = 0; J <= jmax && ok; ++J) {
        const int buf = J & 1;
        const uint32_t acc_phase = (J >> 1) & 1;
        if (!mbar_wait(&sm.acc_empty[buf], acc_phase ^ 1u, abort, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + buf * 256;
        for (int t = 0; t < stages_per_tile; ++t) {
          if (!mbar_wait(&sm.full[stage], phase, abort, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(sm.stage[stage]);
          const uint32_t sb = sa + kBytesA;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = make_sdesc_sw128(sa + kk * 32, 16, 1024);
            const uint64_t bd = make_sdesc_sw128(sb + kk * 32, 16, 1024);
            if constexpr (kFp8) mma_f8_ss(d_tmem, ad, bd, idesc, (t | kk) != 0);
            else mma_bf16_ss(d_tmem, ad, bd, idesc, (t | kk) != 0);
          }
          mma_commit(&sm.empty[stage]);
          if (++stage == kScoreStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) mma_commit(&sm.acc_full[buf]);
      }
      // no MMA may still run when TMEM is released
      mma_commit(&sm.drain);
      mbar_wait(&sm.drain, 0, abort, args.status);
    }
    __syncwarp();
  } else {
    // epilogue: thread owns TMEM lane (query group of the tile) `row`
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    constexpr int gpb = kBlock / s;             // groups per block (16 for s = 8)
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
    constexpr int kbt = kTileN / gpb;    // key blocks per key tile (2 s)
    constexpr int kbc = 32 / gpb;        // key blocks per 32-column chunk
    for (int J = 0; J <= jmax; ++J) {
      const int buf = J & 1;
      // every lane waits; the warp leaves together if any lane gave up
      if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[buf], (J >> 1) & 1, abort, args.status))) break;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t r[32];
        tmem_ld32(tmem + buf * 256 + ch * 32 + (static_cast<uint32_t>(q4 * 32) << 16), r);
        tmem_ld_wait();
        const int b0 = J * kTileN + ch * 32;  // first key group of the chunk
#pragma unroll
        for (int kb = 0; kb < kbc; ++kb) {
          // max over the gpb key groups of this key block (groups past the end excluded) ...
          float v = ninf;
#pragma unroll
          for (int cc = kb * gpb; cc < (kb + 1) * gpb; ++cc)
            v = fmaxf(v, ((b0 + cc) * s < L) ? __uint_as_float(r[cc]) : ninf);
          // ... and over the gpb query groups (consecutive lanes) of each query block
          v = row_valid ? v : ninf;
#pragma unroll
          for (int off = gpb / 2; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          const int j = J * kbt + ch * kbc + kb;
          if (writer && j < args.nb_max) srow[j] = (j <= i) ? fmaf(v, scale, 0.f) + bonus[j] : ninf;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
      if (J == jmax && writer)
        for (int j = (jmax + 1) * kbt; j < args.nb_max; ++j) srow[j] = ninf;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kScoreTmemCols);
  }
}

size_t score_smem_bytes() { return sizeof(ScoreSmem) + 1024; }

template <bool kFp8, int kS>
static cudaError_t launch_score_t(const ScoreMaps& maps, const SeqBatch& batch, const ScoreArgs& args,
                                  cudaStream_t stream) {
  const size_t smem = score_smem_bytes();
  cudaError_t e = cudaFuncSetAttribute(score_kernel<kFp8, kS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  score_kernel<kFp8, kS><<<batch.item0[batch.n], kScoreThreads, smem, stream>>>(maps, batch, args);
  return cudaGetLastError();
}

cudaError_t launch_score(const ScoreMaps& maps, const SeqBatch& batch, const ScoreArgs& args, bool fp8,
                         cudaStream_t stream) {
  if (batch.item0[batch.n] == 0) return cudaSuccess;
  if (args.stride == 8)
    return fp8 ? launch_score_t<true, 8>(maps, batch, args, stream) : launch_score_t<false, 8>(maps, batch, args, stream);
  if (args.stride == 4)
    return fp8 ? launch_score_t<true, 4>(maps, batch, args, stream) : launch_score_t<false, 4>(maps, batch, args, stream);
  return cudaErrorInvalidValue;
}

}  // namespace stem
