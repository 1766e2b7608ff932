// stem_api.cu — the C ABI of include/stem.h: argument validation, planning
// (sizes, nnz, work counts), per-sequence launch batches, TMA descriptor
// encoding and kernel launches.  No allocation, no host<->device copies in
// the compute calls, no synchronisation.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "stem.h"
#include "stem_internal.h"
#include "stem_kernels.h"

using namespace stem;

namespace {

constexpr size_t kStatusBytes = 256;

// An NVTX range over one stage's host-side enqueue (scoring, selection,
// attention), so a timeline profiler shows which launches belong to which
// stage.  Header-only NVTX: without a profiler attached a push/pop is a few
// nanoseconds and loads nothing.
struct StageRange {
  explicit StageRange(const char* name) { nvtxRangePushA(name); }
  ~StageRange() { nvtxRangePop(); }
  StageRange(const StageRange&) = delete;
  StageRange& operator=(const StageRange&) = delete;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct SeqInfo {
  int idx;      // sequence number
  int32_t tok0, len, nb, g0;
  int64_t csr0; // CSR base of the sequence inside one head
};

struct Plan {
  stem_plan_t pub;
  std::vector<SeqInfo> seqs;  // non-empty sequences, longest first
  int B = kBlock;             // block size (tokens): 128, or 64
  size_t off_vbonus, off_vwide, off_scores, off_budgets, off_rowptr, off_colidx;
};

stem_status_t validate(const stem_qkv_t* qkv, const stem_params_t* p) {
  if (!qkv || !p) return STEM_ERR_INVALID_ARG;
  if (qkv->dtype != STEM_BF16 && qkv->dtype != STEM_FP8_E4M3) return STEM_ERR_INVALID_ARG;
  if (qkv->num_seqs < 1 || !qkv->cu_seqlens_host || qkv->total_tokens < 0) return STEM_ERR_INVALID_ARG;
  if (qkv->num_q_heads < 1 || qkv->num_kv_heads < 1 || qkv->num_q_heads % qkv->num_kv_heads != 0)
    return STEM_ERR_INVALID_ARG;
  if (qkv->head_dim != kHeadDim) return qkv->head_dim < 1 ? STEM_ERR_INVALID_ARG : STEM_ERR_UNSUPPORTED;
  const int32_t* cu = qkv->cu_seqlens_host;
  if (cu[0] != 0) return STEM_ERR_INVALID_ARG;
  for (int s = 0; s < qkv->num_seqs; ++s)
    if (cu[s + 1] < cu[s]) return STEM_ERR_INVALID_ARG;
  if (cu[qkv->num_seqs] != qkv->total_tokens) return STEM_ERR_INVALID_ARG;
  if (p->block_size != kBlock && p->block_size != kBlock / 2)
    return p->block_size < 1 ? STEM_ERR_INVALID_ARG : STEM_ERR_UNSUPPORTED;
  if (p->stride < 1 || p->block_size % p->stride != 0) return STEM_ERR_INVALID_ARG;
  if (p->stride != 4 && p->stride != 8) return STEM_ERR_UNSUPPORTED;
  if (p->chunk_size < 1) return STEM_ERR_INVALID_ARG;
  if (!(p->norm > 0.0) || !std::isfinite(p->norm)) return STEM_ERR_INVALID_ARG;
  if (!(p->beta >= 0.0) || !std::isfinite(p->beta)) return STEM_ERR_INVALID_ARG;
  if (!(p->keep_ratio > 0.0 && p->keep_ratio <= 1.0)) return STEM_ERR_INVALID_ARG;
  if (!(p->mu > 0.0 && p->mu <= 1.0)) return STEM_ERR_INVALID_ARG;
  if (p->sink_blocks < 0 || p->window_blocks < 1) return STEM_ERR_INVALID_ARG;
  if (!(p->softmax_scale >= 0.0) || !std::isfinite(p->softmax_scale)) return STEM_ERR_INVALID_ARG;
  if (p->budget_mode != STEM_BUDGET_RELATIVE && p->budget_mode != STEM_BUDGET_ABSOLUTE) return STEM_ERR_INVALID_ARG;
  if (p->bonus_mode != STEM_BONUS_LOG && p->bonus_mode != STEM_BONUS_STANDARDIZED) return STEM_ERR_INVALID_ARG;
  if (p->list_mode != STEM_LIST_PER_HEAD && p->list_mode != STEM_LIST_PER_GROUP) return STEM_ERR_INVALID_ARG;
  if (p->select_mode != STEM_SELECT_SEPARATE && p->select_mode != STEM_SELECT_FUSED) return STEM_ERR_INVALID_ARG;
  return STEM_OK;
}

stem_status_t make_plan(const stem_qkv_t* qkv, const stem_params_t* p, Plan* out) {
  stem_status_t st = validate(qkv, p);
  if (st != STEM_OK) return st;
  const int hq = qkv->num_q_heads, hkv = qkv->num_kv_heads;
  const int s = p->stride, B = p->block_size, gpb = B / s;
  Plan pl{};
  pl.B = B;
  int64_t nbtot = 0, nb_max = 0, nnz_h = 0;
  double pairs_sel = 0, pairs_dense = 0, score_pairs = 0;
  for (int q = 0; q < qkv->num_seqs; ++q) {
    const int32_t o = qkv->cu_seqlens_host[q];
    const int32_t L = qkv->cu_seqlens_host[q + 1] - o;
    const int32_t nb = (L + B - 1) / B;
    if (nb > 0) {
      SeqInfo si{q, o, L, nb, static_cast<int32_t>(nbtot), nnz_h};
      for (int i = 0; i < nb; ++i) {
        const int32_t b = tpd_budget(i, nb, p->keep_ratio, p->mu, p->sink_blocks, p->window_blocks,
                                     p->budget_mode);
        nnz_h += b;
        const double qi = std::min(B, L - i * B);
        pairs_sel += (b - 1) * qi * B + qi * (qi + 1) / 2;
        pairs_dense += static_cast<double>(i) * qi * B + qi * (qi + 1) / 2;
      }
      score_pairs += static_cast<double>(nb) * (nb + 1) / 2 * gpb * gpb;
      pl.seqs.push_back(si);
    }
    nbtot += nb;
    nb_max = std::max<int64_t>(nb_max, nb);
  }
  if (nb_max == 0) nb_max = 1;
  // 64-token blocks: the attention keeps each pair of lists as two bitmaps of
  // kMaxBitmapBlocks bits in shared memory
  if (B != kBlock && nb_max > kMaxBitmapBlocks) return STEM_ERR_UNSUPPORTED;
  const int64_t rows = static_cast<int64_t>(hq) * nbtot;
  const int64_t nnz = nnz_h * hq;
  if (nnz > INT32_MAX || rows + 1 > INT32_MAX) return STEM_ERR_UNSUPPORTED;
  std::stable_sort(pl.seqs.begin(), pl.seqs.end(), [](const SeqInfo& a, const SeqInfo& b) { return a.nb > b.nb; });

  stem_plan_t& pub = pl.pub;
  pub.nb_total = nbtot;
  pub.nb_max = nb_max;
  pub.num_rows = rows;
  pub.nnz = nnz;
  pub.nnz_per_head = nnz_h;
  pub.scores_bytes = static_cast<size_t>(rows) * nb_max * sizeof(float);
  pub.vbonus_bytes = static_cast<size_t>(hkv) * nbtot * sizeof(float);
  // fp8: the attention kernel reads V widened to f16 [T, Hkv, d]
  pub.vwide_bytes = qkv->dtype == STEM_FP8_E4M3
                        ? static_cast<size_t>(qkv->total_tokens) * hkv * kHeadDim * sizeof(uint16_t)
                        : 0;
  pl.off_vbonus = kStatusBytes;
  pl.off_vwide = pl.off_vbonus + align256(pub.vbonus_bytes);
  pub.ws_bytes = pl.off_vwide + align256(pub.vwide_bytes);
  pl.off_scores = pub.ws_bytes;
  pl.off_budgets = pl.off_scores + align256(pub.scores_bytes);
  pl.off_rowptr = pl.off_budgets + align256(static_cast<size_t>(rows) * 4);
  pl.off_colidx = pl.off_rowptr + align256(static_cast<size_t>(rows + 1) * 4);
  pub.ws_prefill_bytes = pl.off_colidx + align256(static_cast<size_t>(nnz) * 4);
  pub.attn_flops = 4.0 * kHeadDim * hq * pairs_sel;
  pub.dense_attn_flops = 4.0 * kHeadDim * hq * pairs_dense;
  pub.score_flops = 2.0 * s * kHeadDim * hq * score_pairs;
  *out = std::move(pl);
  return STEM_OK;
}

stem_status_t check_tensors(const stem_qkv_t* qkv) {
  if (qkv->total_tokens > 0) {
    if (!qkv->q || !qkv->k || !qkv->v || !qkv->cu_seqlens) return STEM_ERR_INVALID_ARG;
    if (!aligned16(qkv->q) || !aligned16(qkv->k) || !aligned16(qkv->v)) return STEM_ERR_MISALIGNED;
  }
  if (qkv->dtype == STEM_FP8_E4M3 && (!qkv->q_scale || !qkv->k_scale || !qkv->v_scale)) return STEM_ERR_INVALID_ARG;
  return STEM_OK;
}

// Split the non-empty sequences into launch batches of at most
// kMaxSeqPerLaunch; items(si) is the number of CTAs a sequence needs.
template <class F>
std::vector<SeqBatch> make_batches(const Plan& pl, F items) {
  std::vector<SeqBatch> out;
  for (size_t b0 = 0; b0 < pl.seqs.size(); b0 += kMaxSeqPerLaunch) {
    SeqBatch b{};
    b.n = static_cast<int32_t>(std::min<size_t>(kMaxSeqPerLaunch, pl.seqs.size() - b0));
    b.item0[0] = 0;
    for (int q = 0; q < b.n; ++q) {
      const SeqInfo& si = pl.seqs[b0 + q];
      b.tok0[q] = si.tok0;
      b.len[q] = si.len;
      b.nb[q] = si.nb;
      b.g0[q] = si.g0;
      b.csr0[q] = si.csr0;
      b.seq_id[q] = si.idx;
      b.item0[q + 1] = b.item0[q] + items(si);
    }
    for (int q = b.n; q < kMaxSeqPerLaunch; ++q) b.item0[q + 1] = b.item0[q];
    out.push_back(b);
  }
  return out;
}

// ---------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 3-D map over one sequence of a [T, H, 128] tensor: dims (d, head, token),
// box (inner, 1, box_tokens) traversed with token stride `tstride`, 128-B swizzle.
// The len / s full groups of s tokens of one sequence as a 4-d tensor
// (dim, head, slot u, group g) -> token g s + u; box (one 128-B slab, 1, 1,
// box_groups): one copy brings slot u of box_groups consecutive groups.  Only
// whole groups are mapped, so no copy reads past the sequence; groups beyond
// are zero-filled.  False when the sequence has no whole group.
bool encode_group_map(CUtensorMap* m, const void* base, bool fp8, int heads, int tok0, int len, int s,
                      int box_groups) {
  EncodeTiledFn fn = encode_fn();
  if (!fn || len / s == 0) return false;
  const size_t elt = fp8 ? 1 : 2;
  const size_t row = static_cast<size_t>(heads) * kHeadDim * elt;  // bytes per token
  const uint8_t* b = static_cast<const uint8_t*>(base) + static_cast<size_t>(tok0) * row;
  cuuint64_t dims[4] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(s), static_cast<cuuint64_t>(len / s)};
  cuuint64_t strides[3] = {static_cast<cuuint64_t>(kHeadDim * elt), static_cast<cuuint64_t>(row),
                           static_cast<cuuint64_t>(row * s)};
  cuuint32_t box[4] = {static_cast<cuuint32_t>(fp8 ? 128 : 64), 1u, 1u, static_cast<cuuint32_t>(box_groups)};
  cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
  CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
                  const_cast<uint8_t*>(b), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_seq_map(CUtensorMap* m, const void* base, bool fp8, int heads, int tok0, int len, int box_tokens,
                    int tstride) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const size_t elt = fp8 ? 1 : 2;
  const uint8_t* b = static_cast<const uint8_t*>(base) + static_cast<size_t>(tok0) * heads * kHeadDim * elt;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(heads),
                        static_cast<cuuint64_t>(len)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim * elt), static_cast<cuuint64_t>(heads * kHeadDim * elt)};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(fp8 ? 128 : 64), 1u, static_cast<cuuint32_t>(box_tokens)};
  cuuint32_t estr[3] = {1u, 1u, static_cast<cuuint32_t>(tstride)};
  CUresult r = fn(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<uint8_t*>(b), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

stem_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? STEM_OK : STEM_ERR_CUDA; }

double sm_scale(const stem_params_t* p) {
  return p->softmax_scale > 0.0 ? p->softmax_scale : 1.0 / std::sqrt(static_cast<double>(kHeadDim));
}

// ---------------------------------------------------------------- stages
// Every run_* below handles the KV heads hk0 .. hk0 + nhk - 1 (and their query
// heads) only, so a caller can work through a layer one KV-head group at a time.
// With budgets / row_ptr / col_idx given (fused selection), the budgets must
// already be complete: the scoring CTAs then also write the lists.
stem_status_t run_score(const stem_qkv_t* qkv, const stem_params_t* p, const Plan& pl, int hk0, int nhk, float* scores,
                        float* vbonus, int* status, cudaStream_t stream, const int32_t* budgets = nullptr,
                        const int32_t* row_ptr = nullptr, int32_t* col_idx = nullptr) {
  StageRange nvtx_range("stem: score");
  const bool fp8 = qkv->dtype == STEM_FP8_E4M3;
  const int hq = qkv->num_q_heads, hkv = qkv->num_kv_heads, s = p->stride;
  const int nbtot = static_cast<int>(pl.pub.nb_total), nb_max = static_cast<int>(pl.pub.nb_max);
  for (const SeqBatch& b : make_batches(pl, [](const SeqInfo& si) { return si.nb; })) {
    stem_status_t st = cuda_status(
        launch_vnorm(b, qkv->v, qkv->v_scale, fp8, hkv, hk0, nhk, nbtot, pl.B, static_cast<float>(p->beta),
                     p->bonus_mode == STEM_BONUS_STANDARDIZED, vbonus, stream));
    if (st != STEM_OK) return st;
  }
  // standardized bonus: z-score over each sequence's blocks, per KV head
  for (const SeqBatch& b : make_batches(pl, [&](const SeqInfo&) { return nhk; })) {
    if (p->bonus_mode != STEM_BONUS_STANDARDIZED) break;
    stem_status_t st = cuda_status(launch_bonus_standardize(b, hk0, nbtot, static_cast<float>(p->beta), vbonus, stream));
    if (st != STEM_OK) return st;
  }
  ScoreArgs a{};
  a.hq = hq;
  a.hkv = hkv;
  a.nbtot = nbtot;
  a.nb_max = nb_max;
  a.stride = s;
  a.block = pl.B;
  a.scale = static_cast<float>(1.0 / (std::sqrt(static_cast<double>(kHeadDim)) * s * p->norm));
  a.q_scale = qkv->q_scale;
  a.k_scale = qkv->k_scale;
  a.vbonus = vbonus;
  a.scores = scores;
  a.status = status;
  a.hk0 = hk0;
  a.fuse_select = budgets != nullptr;
  a.sink = p->sink_blocks;
  a.window = p->window_blocks;
  a.budgets = budgets;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  // one CTA per (pair of query heads of a KV group, 128-group query tile of
  // 128 s / B query blocks)
  const int pairs = nhk * ((hq / hkv + 1) / 2);
  const int blocks_per_tile = 128 * s / pl.B;
  for (const SeqBatch& b : make_batches(pl, [&](const SeqInfo& si) {
         return pairs * ((si.nb + blocks_per_tile - 1) / blocks_per_tile);
       })) {
    ScoreMaps maps;
    std::memset(&maps, 0, sizeof(maps));
    for (int q = 0; q < b.n; ++q) {
      if (!encode_seq_map(&maps.q[q], qkv->q, fp8, hq, b.tok0[q], b.len[q], 256, s) ||
          !encode_seq_map(&maps.k[q], qkv->k, fp8, hkv, b.tok0[q], b.len[q], 256, s))
        return STEM_ERR_CUDA;
      maps.group_maps[q] = b.len[q] / s > 0;
      if (maps.group_maps[q] && (!encode_group_map(&maps.q_groups[q], qkv->q, fp8, hq, b.tok0[q], b.len[q], s, 128) ||
                                 !encode_group_map(&maps.k_groups[q], qkv->k, fp8, hkv, b.tok0[q], b.len[q], s, 256)))
        return STEM_ERR_CUDA;
    }
    stem_status_t st = cuda_status(launch_score(maps, b, a, fp8, stream));
    if (st != STEM_OK) return st;
  }
  return STEM_OK;
}

// The scoring kernel selects the rows it scored (no separate selection pass)
// when asked to, for per-head lists whose rows fit its scratch.  Separate is
// the default: one warp per list over every list at once finishes sooner
// than each scoring CTA selecting its own rows after its last key tile.
bool fuse_selection(const stem_params_t* p, const Plan& pl) {
  return p->select_mode == STEM_SELECT_FUSED && p->list_mode == STEM_LIST_PER_HEAD &&
         pl.pub.nb_max <= kFusedSelectMaxBlocks;
}

stem_status_t run_select(const stem_qkv_t* qkv, const stem_params_t* p, const Plan& pl, int hk0, int nhk,
                         bool with_budgets, const float* scores,
                         int32_t* budgets, int32_t* row_ptr, int32_t* col_idx, cudaStream_t stream,
                         bool with_lists = true) {
  StageRange nvtx_range("stem: select");
  const int hq = qkv->num_q_heads;
  const int nbtot = static_cast<int>(pl.pub.nb_total), nb_max = static_cast<int>(pl.pub.nb_max);
  const int G = hq / qkv->num_kv_heads;
  for (const SeqBatch& b : make_batches(pl, [](const SeqInfo&) { return 1; })) {
    if (!with_budgets) break;
    stem_status_t st = cuda_status(launch_budget(b, hq, nbtot, pl.pub.nnz_per_head, p->keep_ratio, p->mu,
                                                 p->sink_blocks, p->window_blocks, p->budget_mode, budgets,
                                                 row_ptr, stream));
    if (st != STEM_OK) return st;
  }
  // one CTA per list: per (query head, query block), or per (KV head, query
  // block) when the query heads of a group share their lists
  const int per_list = p->list_mode == STEM_LIST_PER_GROUP ? G : 1;
  for (const SeqBatch& b : make_batches(pl, [&](const SeqInfo& si) { return nhk * (G / per_list) * si.nb; })) {
    if (!with_lists) break;
    stem_status_t st = cuda_status(launch_select(b, hq, hk0 * G, nhk * G, per_list, nbtot, nb_max, p->sink_blocks,
                                                 p->window_blocks, scores,
                                                 budgets, row_ptr, col_idx, stream));
    if (st != STEM_OK) return st;
  }
  return STEM_OK;
}

// ws: the call's workspace (status word first, the widened V at off_vwide).
stem_status_t run_bsa(const stem_qkv_t* qkv, const stem_params_t* p, const Plan& pl, int hk0, int nhk,
                      const int32_t* row_ptr, const int32_t* col_idx, void* out, float* lse, void* ws,
                      cudaStream_t stream, const stem_paged_kv_t* paged = nullptr) {
  StageRange nvtx_range("stem: attention");
  const bool fp8 = qkv->dtype == STEM_FP8_E4M3;
  const int hq = qkv->num_q_heads, hkv = qkv->num_kv_heads;
  int* status = static_cast<int*>(ws);
  uint16_t* v16 = reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(ws) + pl.off_vwide);
  if (fp8) {
    // V of these KV heads widened to f16, packed (gathered through the page
    // table for paged K/V)
    stem_status_t st = cuda_status(
        paged ? launch_vwiden(paged->v_pages, v16, qkv->total_tokens, hkv, hk0, nhk, qkv->cu_seqlens,
                              qkv->num_seqs, paged->page_table, paged->page_size, paged->num_pages,
                              paged->max_pages_per_seq, stream)
              : launch_vwiden(qkv->v, v16, qkv->total_tokens, hkv, hk0, nhk, nullptr, qkv->num_seqs, nullptr, 0,
                              0, 0, stream));
    if (st != STEM_OK) return st;
  }
  BsaArgs a{};
  a.hq = hq;
  a.hkv = hkv;
  a.nbtot = static_cast<int>(pl.pub.nb_total);
  a.total_tokens = qkv->total_tokens;
  a.scale_log2 = static_cast<float>(sm_scale(p) * 1.4426950408889634);
  a.q_scale = qkv->q_scale;
  a.k_scale = qkv->k_scale;
  a.v_scale = qkv->v_scale;
  a.row_ptr = row_ptr;
  a.col_idx = col_idx;
  a.q = qkv->q;
  a.out = out;
  a.lse = lse;
  a.status = status;
  a.hk0 = hk0;
  a.block = pl.B;
  BsaMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (paged) {
    // the page pool as one token sequence of pages * page_size rows
    const int pool = paged->num_pages * paged->page_size;
    if (!encode_seq_map(&maps.k_pool, paged->k_pages, fp8, hkv, 0, pool, kBlock / 2, 1) ||
        (!fp8 && !encode_seq_map(&maps.v_pool, paged->v_pages, false, hkv, 0, pool, kBlock / 2, 1)))
      return STEM_ERR_CUDA;
    a.page_table = paged->page_table;
    a.page_size = paged->page_size;
    a.max_pages = paged->max_pages_per_seq;
  }
  // one CTA per CSR row (query head, query block), or, with lists shared by
  // the query heads of a group, per (query block, pair of query heads); with
  // 64-token blocks one CTA per query head and pair of query blocks (one
  // 128-token query tile)
  const int G = hq / hkv;
  const bool pairs = p->list_mode == STEM_LIST_PER_GROUP && G >= 2 && pl.B == kBlock;
  for (const SeqBatch& b : make_batches(pl, [&](const SeqInfo& si) {
         const int tiles = pl.B == kBlock ? si.nb : (si.nb + 1) / 2;
         return pairs ? nhk * ((G + 1) / 2) * tiles : nhk * G * tiles;
       })) {
    for (int q = 0; q < b.n; ++q) {
      // Q in 128-token boxes; K and V in 64-token boxes (the attention
      // kernel moves half a key block per copy)
      if (!encode_seq_map(&maps.q[q], qkv->q, fp8, hq, b.tok0[q], b.len[q], kBlock, 1)) return STEM_ERR_CUDA;
      if (!paged && !encode_seq_map(&maps.k[q], qkv->k, fp8, hkv, b.tok0[q], b.len[q], kBlock / 2, 1))
        return STEM_ERR_CUDA;
      // V: the widened f16 copy (fp8), or the bf16 input when not paged
      if ((fp8 || !paged) &&
          !encode_seq_map(&maps.v[q], fp8 ? static_cast<const void*>(v16) : qkv->v, false, hkv, b.tok0[q], b.len[q],
                          kBlock / 2, 1))
        return STEM_ERR_CUDA;
    }
    stem_status_t st =
        cuda_status(pairs ? launch_bsa_pair(maps, b, a, fp8, stream) : launch_bsa(maps, b, a, fp8, stream));
    if (st != STEM_OK) return st;
  }
  return STEM_OK;
}

stem_status_t clear_status(void* ws, cudaStream_t stream) {
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(int), stream));
}

}  // namespace

extern "C" {

stem_status_t stem_plan(const stem_qkv_t* qkv, const stem_params_t* params, stem_plan_t* out) {
  if (!out) return STEM_ERR_INVALID_ARG;
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st == STEM_OK) *out = pl.pub;
  return st;
}

stem_status_t stem_score(const stem_qkv_t* qkv, const stem_params_t* params, float* scores, float* vbonus,
                         void* ws, size_t ws_bytes, stem_stream_t stream) {
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if ((st = check_tensors(qkv)) != STEM_OK) return st;
  if (!scores || !ws) return STEM_ERR_INVALID_ARG;
  if (ws_bytes < pl.pub.ws_bytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != STEM_OK) return st;
  float* vb = vbonus ? vbonus : reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_vbonus);
  return run_score(qkv, params, pl, 0, qkv->num_kv_heads, scores, vb, static_cast<int*>(ws), s);
}

stem_status_t stem_score_select(const stem_qkv_t* qkv, const stem_params_t* params, float* scores, float* vbonus,
                                int32_t* budgets, int32_t* row_ptr, int32_t* col_idx, void* ws, size_t ws_bytes,
                                stem_stream_t stream) {
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if ((st = check_tensors(qkv)) != STEM_OK) return st;
  if (!scores || !budgets || !row_ptr || !ws || (!col_idx && pl.pub.nnz > 0)) return STEM_ERR_INVALID_ARG;
  if (ws_bytes < pl.pub.ws_bytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != STEM_OK) return st;
  float* vb = vbonus ? vbonus : reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.off_vbonus);
  int* status = static_cast<int*>(ws);
  const int hkv = qkv->num_kv_heads;
  if (fuse_selection(params, pl)) {
    if ((st = run_select(qkv, params, pl, 0, hkv, true, scores, budgets, row_ptr, col_idx, s, false)) != STEM_OK)
      return st;
    return run_score(qkv, params, pl, 0, hkv, scores, vb, status, s, budgets, row_ptr, col_idx);
  }
  if ((st = run_score(qkv, params, pl, 0, hkv, scores, vb, status, s)) != STEM_OK) return st;
  return run_select(qkv, params, pl, 0, hkv, true, scores, budgets, row_ptr, col_idx, s);
}

stem_status_t stem_select(const stem_qkv_t* qkv, const stem_params_t* params, const float* scores,
                          int32_t* budgets, int32_t* row_ptr, int32_t* col_idx, void* ws, size_t ws_bytes,
                          stem_stream_t stream) {
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if (!scores || !budgets || !row_ptr || !ws || (!col_idx && pl.pub.nnz > 0)) return STEM_ERR_INVALID_ARG;
  if (ws_bytes < pl.pub.ws_bytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != STEM_OK) return st;
  return run_select(qkv, params, pl, 0, qkv->num_kv_heads, true, scores, budgets, row_ptr, col_idx, s);
}

stem_status_t stem_bsa_fwd(const stem_qkv_t* qkv, const stem_params_t* params, const int32_t* row_ptr,
                           const int32_t* col_idx, void* out, float* lse, void* ws, size_t ws_bytes,
                           stem_stream_t stream) {
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if ((st = check_tensors(qkv)) != STEM_OK) return st;
  if (!row_ptr || !col_idx || !out || !lse || !ws) return STEM_ERR_INVALID_ARG;
  if (!aligned16(out)) return STEM_ERR_MISALIGNED;
  if (ws_bytes < pl.pub.ws_bytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != STEM_OK) return st;
  return run_bsa(qkv, params, pl, 0, qkv->num_kv_heads, row_ptr, col_idx, out, lse, ws, s);
}

stem_status_t stem_bsa_fwd_paged(const stem_qkv_t* qkv, const stem_paged_kv_t* kv, const stem_params_t* params,
                                 const int32_t* row_ptr, const int32_t* col_idx, void* out, float* lse, void* ws,
                                 size_t ws_bytes, stem_stream_t stream) {
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if (!kv) return STEM_ERR_INVALID_ARG;
  if (qkv->total_tokens > 0) {
    if (!qkv->q || !qkv->cu_seqlens || !kv->k_pages || !kv->v_pages || !kv->page_table) return STEM_ERR_INVALID_ARG;
    if (!aligned16(qkv->q) || !aligned16(kv->k_pages) || !aligned16(kv->v_pages)) return STEM_ERR_MISALIGNED;
  }
  if (qkv->dtype == STEM_FP8_E4M3 && (!qkv->q_scale || !qkv->k_scale || !qkv->v_scale)) return STEM_ERR_INVALID_ARG;
  // a 64-key half must sit inside one page, and every token needs a page
  if (kv->page_size < 64 || kv->page_size % 64 != 0 || kv->num_pages < 1 || kv->max_pages_per_seq < 1)
    return STEM_ERR_INVALID_ARG;
  if (static_cast<int64_t>(kv->num_pages) * kv->page_size > INT32_MAX) return STEM_ERR_INVALID_ARG;
  for (int q = 0; q < qkv->num_seqs; ++q) {
    const int64_t L = qkv->cu_seqlens_host[q + 1] - qkv->cu_seqlens_host[q];
    // the last key block may run past L to its end (a multiple of the block size)
    const int64_t need = (L + params->block_size - 1) / params->block_size * params->block_size;
    if (need > static_cast<int64_t>(kv->max_pages_per_seq) * kv->page_size) return STEM_ERR_INVALID_ARG;
  }
  if (!row_ptr || !col_idx || !out || !lse || !ws) return STEM_ERR_INVALID_ARG;
  if (!aligned16(out)) return STEM_ERR_MISALIGNED;
  if (ws_bytes < pl.pub.ws_bytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if ((st = clear_status(ws, s)) != STEM_OK) return st;
  return run_bsa(qkv, params, pl, 0, qkv->num_kv_heads, row_ptr, col_idx, out, lse, ws, s, kv);
}

stem_status_t stem_prefill(const stem_qkv_t* qkv, const stem_params_t* params, void* out, float* lse,
                           int32_t* row_ptr_out, int32_t* col_idx_out, void* ws, size_t ws_bytes,
                           stem_stream_t stream) {
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if ((st = check_tensors(qkv)) != STEM_OK) return st;
  if (!out || !lse || !ws) return STEM_ERR_INVALID_ARG;
  if (!aligned16(out)) return STEM_ERR_MISALIGNED;
  if (ws_bytes < pl.pub.ws_prefill_bytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(w);
  float* vbonus = reinterpret_cast<float*>(w + pl.off_vbonus);
  float* scores = reinterpret_cast<float*>(w + pl.off_scores);
  int32_t* budgets = reinterpret_cast<int32_t*>(w + pl.off_budgets);
  int32_t* row_ptr = row_ptr_out ? row_ptr_out : reinterpret_cast<int32_t*>(w + pl.off_rowptr);
  int32_t* col_idx = col_idx_out ? col_idx_out : reinterpret_cast<int32_t*>(w + pl.off_colidx);
  if ((st = clear_status(ws, s)) != STEM_OK) return st;
  const int hkv = qkv->num_kv_heads;
  if (fuse_selection(params, pl)) {
    // budgets first; the scoring CTAs then select the rows they scored
    if ((st = run_select(qkv, params, pl, 0, hkv, true, scores, budgets, row_ptr, col_idx, s, false)) != STEM_OK ||
        (st = run_score(qkv, params, pl, 0, hkv, scores, vbonus, status, s, budgets, row_ptr, col_idx)) != STEM_OK)
      return st;
  } else {
    if ((st = run_score(qkv, params, pl, 0, hkv, scores, vbonus, status, s)) != STEM_OK) return st;
    if ((st = run_select(qkv, params, pl, 0, hkv, true, scores, budgets, row_ptr, col_idx, s)) != STEM_OK) return st;
  }
  return run_bsa(qkv, params, pl, 0, hkv, row_ptr, col_idx, out, lse, ws, s);
}

stem_status_t stem_prefill_host(const stem_qkv_t* qkv, const stem_params_t* params, const void* q_host,
                                const void* k_host, const void* v_host, void* out_dev, float* lse_dev,
                                void* out_host, float* lse_host, void* ws, size_t ws_bytes, stem_stream_t stream) {
  Plan pl;
  stem_status_t st = make_plan(qkv, params, &pl);
  if (st != STEM_OK) return st;
  if ((st = check_tensors(qkv)) != STEM_OK) return st;
  if (!q_host || !k_host || !v_host || !out_dev || !lse_dev || !out_host || !lse_host || !ws)
    return STEM_ERR_INVALID_ARG;
  if (!aligned16(out_dev)) return STEM_ERR_MISALIGNED;
  if (ws_bytes < pl.pub.ws_prefill_bytes) return STEM_ERR_WORKSPACE_TOO_SMALL;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(w);
  float* vbonus = reinterpret_cast<float*>(w + pl.off_vbonus);
  float* scores = reinterpret_cast<float*>(w + pl.off_scores);
  int32_t* budgets = reinterpret_cast<int32_t*>(w + pl.off_budgets);
  int32_t* row_ptr = reinterpret_cast<int32_t*>(w + pl.off_rowptr);
  int32_t* col_idx = reinterpret_cast<int32_t*>(w + pl.off_colidx);

  const int hq = qkv->num_q_heads, hkv = qkv->num_kv_heads, G = hq / hkv;
  const size_t T = static_cast<size_t>(qkv->total_tokens);
  const size_t elt = qkv->dtype == STEM_FP8_E4M3 ? 1 : 2;
  const size_t dq = static_cast<size_t>(kHeadDim) * elt;  // bytes of one head row
  const int ngroups = hkv < 8 ? hkv : 8;
  const int per = (hkv + ngroups - 1) / ngroups;  // KV heads per group (the last may have fewer)

  // a copy-in and a copy-out stream and the events that chain them with `s`;
  // released at once: they are freed when the work they order has completed
  cudaStream_t cin = nullptr, cout = nullptr;
  cudaEvent_t ev_begin = nullptr, ev_done = nullptr, ev_in[8] = {}, ev_comp[8] = {};
  auto release = [&]() {
    if (cin) cudaStreamDestroy(cin);
    if (cout) cudaStreamDestroy(cout);
    if (ev_begin) cudaEventDestroy(ev_begin);
    if (ev_done) cudaEventDestroy(ev_done);
    for (int g = 0; g < 8; ++g) {
      if (ev_in[g]) cudaEventDestroy(ev_in[g]);
      if (ev_comp[g]) cudaEventDestroy(ev_comp[g]);
    }
  };
  auto fail = [&](cudaError_t e) {
    release();
    return cuda_status(e);
  };
  cudaError_t e = cudaStreamCreateWithFlags(&cin, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&cout, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_begin, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_done, cudaEventDisableTiming);
  for (int g = 0; g < ngroups && e == cudaSuccess; ++g) {
    e = cudaEventCreateWithFlags(&ev_in[g], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_comp[g], cudaEventDisableTiming);
  }
  if (e != cudaSuccess) return fail(e);

  // inputs: one 2-d copy per tensor and group (the group's heads are a slab of
  // every token row)
  if ((e = cudaEventRecord(ev_begin, s)) != cudaSuccess || (e = cudaStreamWaitEvent(cin, ev_begin, 0)) != cudaSuccess)
    return fail(e);
  for (int g = 0; g < ngroups; ++g) {
    const int hk0 = g * per, nhk = (hk0 + per <= hkv) ? per : hkv - hk0;
    if (nhk <= 0) break;
    const size_t oq = static_cast<size_t>(hk0) * G * dq, ok = static_cast<size_t>(hk0) * dq;
    e = cudaMemcpy2DAsync(static_cast<uint8_t*>(const_cast<void*>(qkv->q)) + oq, hq * dq, static_cast<const uint8_t*>(q_host) + oq,
                          hq * dq, nhk * G * dq, T, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(static_cast<uint8_t*>(const_cast<void*>(qkv->k)) + ok, hkv * dq, static_cast<const uint8_t*>(k_host) + ok,
                            hkv * dq, nhk * dq, T, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(static_cast<uint8_t*>(const_cast<void*>(qkv->v)) + ok, hkv * dq, static_cast<const uint8_t*>(v_host) + ok,
                            hkv * dq, nhk * dq, T, cudaMemcpyHostToDevice, cin);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[g], cin);
    if (e != cudaSuccess) return fail(e);
  }
  // compute on `s`, group by group; results back on the copy-out stream
  if ((st = clear_status(ws, s)) != STEM_OK) {
    release();
    return st;
  }
  for (int g = 0; g < ngroups; ++g) {
    const int hk0 = g * per, nhk = (hk0 + per <= hkv) ? per : hkv - hk0;
    if (nhk <= 0) break;
    if ((e = cudaStreamWaitEvent(s, ev_in[g], 0)) != cudaSuccess) return fail(e);
    const bool fused = fuse_selection(params, pl);
    if (fused) {
      // budgets (all heads) before the first group's scoring, which selects too
      if ((g == 0 &&
           (st = run_select(qkv, params, pl, hk0, nhk, true, scores, budgets, row_ptr, col_idx, s, false)) != STEM_OK) ||
          (st = run_score(qkv, params, pl, hk0, nhk, scores, vbonus, status, s, budgets, row_ptr, col_idx)) != STEM_OK) {
        release();
        return st;
      }
    } else if ((st = run_score(qkv, params, pl, hk0, nhk, scores, vbonus, status, s)) != STEM_OK ||
               (st = run_select(qkv, params, pl, hk0, nhk, g == 0, scores, budgets, row_ptr, col_idx, s)) != STEM_OK) {
      release();
      return st;
    }
    if ((st = run_bsa(qkv, params, pl, hk0, nhk, row_ptr, col_idx, out_dev, lse_dev, ws, s)) != STEM_OK) {
      release();
      return st;
    }
    if ((e = cudaEventRecord(ev_comp[g], s)) != cudaSuccess || (e = cudaStreamWaitEvent(cout, ev_comp[g], 0)) != cudaSuccess)
      return fail(e);
    const size_t oo = static_cast<size_t>(hk0) * G * kHeadDim * 2;  // O is bf16
    e = cudaMemcpy2DAsync(static_cast<uint8_t*>(out_host) + oo, hq * kHeadDim * 2,
                          static_cast<const uint8_t*>(out_dev) + oo, hq * kHeadDim * 2, nhk * G * kHeadDim * 2, T,
                          cudaMemcpyDeviceToHost, cout);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(lse_host + static_cast<size_t>(hk0) * G * T, lse_dev + static_cast<size_t>(hk0) * G * T,
                          static_cast<size_t>(nhk) * G * T * sizeof(float), cudaMemcpyDeviceToHost, cout);
    if (e != cudaSuccess) return fail(e);
  }
  if ((e = cudaEventRecord(ev_done, cout)) != cudaSuccess || (e = cudaStreamWaitEvent(s, ev_done, 0)) != cudaSuccess)
    return fail(e);
  release();
  return STEM_OK;
}

stem_status_t stem_read_device_status(const void* ws, stem_stream_t stream, stem_status_t* out) {
  if (!ws || !out) return STEM_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return STEM_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return STEM_ERR_CUDA;
  *out = static_cast<stem_status_t>(v);
  return STEM_OK;
}

const char* stem_status_string(stem_status_t status) {
  switch (status) {
    case STEM_OK: return "ok";
    case STEM_ERR_INVALID_ARG: return "invalid argument";
    case STEM_ERR_UNSUPPORTED: return "unsupported configuration";
    case STEM_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case STEM_ERR_MISALIGNED: return "tensor pointer not 16-byte aligned";
    case STEM_ERR_CUDA: return "CUDA error";
    case STEM_ERR_TIMEOUT: return "device pipeline wait timed out";
    case STEM_ERR_BAD_BLOCKLIST: return "malformed block list entry skipped";
  }
  return "unknown status";
}

int32_t stem_version(void) { return 100; }

}  // extern "C"
