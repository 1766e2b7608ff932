// stem_kernels.h — kernel launch interfaces used by the host API (stem_api.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "stem_internal.h"

namespace stem {

// Per-sequence TMA descriptors of one launch (kernel parameters, so the
// kernels need no descriptor copies in global memory).
struct ScoreMaps {
  CUtensorMap q[kMaxSeqPerLaunch];  // token traversal stride s, box 256 tokens
  CUtensorMap k[kMaxSeqPerLaunch];
  // the full s-token groups of a sequence as (dim, head, slot, group), box of
  // 128 (q) or 256 (k) groups of one slot; valid where group_maps[seq] != 0
  CUtensorMap q_groups[kMaxSeqPerLaunch];
  CUtensorMap k_groups[kMaxSeqPerLaunch];
  int group_maps[kMaxSeqPerLaunch];
};

struct BsaMaps {
  CUtensorMap q[kMaxSeqPerLaunch];  // box 128 tokens
  CUtensorMap k[kMaxSeqPerLaunch];  // box 64 tokens (unused when K/V are paged)
  CUtensorMap v[kMaxSeqPerLaunch];
  CUtensorMap k_pool;               // paged K/V: the whole page pool as [pages * page_size] tokens
  CUtensorMap v_pool;
};

struct ScoreArgs {
  int hq, hkv, nbtot, nb_max, stride;
  int block;                // block size (tokens): 128 or 64
  int hk0;                  // first KV head of the launch (its items cover consecutive KV heads)
  int num_sms;              // SMs of the device (the CTA order depends on it, never the results)
  float scale;              // 1 / (sqrt(d) s n)
  const float* q_scale;     // fp8 only
  const float* k_scale;
  const float* vbonus;      // [Hkv][NBtot]
  float* scores;            // [Hq][NBtot][nb_max]
  int* status;
  // fused selection: when set, every CTA also selects the rows it scored
  // (budgets and row_ptr must be complete; nb_max <= kFusedSelectMaxBlocks)
  int fuse_select;
  int sink, window;
  const int32_t* budgets;
  const int32_t* row_ptr;
  int32_t* col_idx;
};
// largest nb_max for which the scoring kernel can select its rows itself (the
// per-warp selection scratch lives in the drained operand stages)
constexpr int kFusedSelectMaxBlocks = 5888;

struct BsaArgs {
  int hq, hkv, nbtot, total_tokens;
  int block;                // block size (tokens): 128, or 64 (one CTA then covers query blocks 2p and 2p + 1)
  int hk0;                  // first KV head of the launch (its items cover consecutive KV heads)
  const int32_t* page_table;  // paged K/V: [num_seqs][max_pages] physical page per logical page, else null
  int page_size;            // tokens per page, a multiple of 64
  int max_pages;            // row length of page_table
  float scale_log2;         // softmax scale * log2(e)
  const float* q_scale;     // fp8 only
  const float* k_scale;
  const float* v_scale;
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const void* q;            // [T, Hq, d] (rows are read straight into TMEM)
  void* out;                // bf16 [T, Hq, d]
  float* lse;               // [Hq][T]
  int* status;
};

// KV heads hk0 .. hk0 + nhk - 1 only.  raw_log: write x = ln max ||v||^2 for a
// later launch_bonus_standardize instead of beta * max(0, x).
cudaError_t launch_vnorm(const SeqBatch& batch, const void* v, const float* v_scale, bool fp8, int hkv, int hk0,
                         int nhk, int nbtot, int block, float beta, bool raw_log, float* vbonus,
                         cudaStream_t stream);
// vbonus[hk][g] = beta * max(0, (x - mean) / std) over the finite x of each
// sequence, for KV heads hk0 .. hk0 + (items per sequence) - 1.
cudaError_t launch_bonus_standardize(const SeqBatch& batch, int hk0, int nbtot, float beta, float* vbonus,
                                     cudaStream_t stream);
cudaError_t launch_score(const ScoreMaps& maps, const SeqBatch& batch, const ScoreArgs& args, bool fp8,
                         cudaStream_t stream);
cudaError_t launch_budget(const SeqBatch& batch, int hq, int nbtot, int64_t nnz_per_head, double rho, double mu,
                          int sink, int window, int mode, int32_t* budgets, int32_t* row_ptr, cudaStream_t stream);
// rows of query heads h0 .. h0 + nh - 1 only; `group` consecutive heads share
// one list selected on the max of their scores (batch items: nh / group * nb
// per sequence)
cudaError_t launch_select(const SeqBatch& batch, int hq, int h0, int nh, int group, int nbtot, int nb_max, int sink,
                          int window,
                          const float* scores, const int32_t* budgets, const int32_t* row_ptr, int32_t* col_idx,
                          cudaStream_t stream);
cudaError_t launch_bsa(const BsaMaps& maps, const SeqBatch& batch, const BsaArgs& args, bool fp8,
                       cudaStream_t stream);
// Rows whose lists are shared by the query heads of a KV group: one CTA per
// (query block, pair of query heads), K and V staged once for the pair
// (batch items: nhk * ceil(G / 2) * nb per sequence).
cudaError_t launch_bsa_pair(const BsaMaps& maps, const SeqBatch& batch, const BsaArgs& args, bool fp8,
                            cudaStream_t stream);
// fp8 V widened to f16 rows [T, Hkv, d] for KV heads hk0 .. hk0 + nhk - 1, read
// packed or (page_table non-null) through the page table.
cudaError_t launch_vwiden(const void* v8, uint16_t* v16, int total_tokens, int hkv, int hk0, int nhk,
                          const int32_t* cu_seqlens, int num_seqs, const int32_t* page_table, int page_size,
                          int num_pages, int max_pages, cudaStream_t stream);

size_t score_smem_bytes();
size_t bsa_smem_bytes(bool fp8);

}  // namespace stem
