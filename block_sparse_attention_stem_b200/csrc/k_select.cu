// k_select.cu — token position-decay budgets, CSR row pointers and the top-k
// block selection.
//
// Budget: "Stem" gist.science zh summary §2.1, k(i) = floor(k_start -
// k_start (1-mu)/N * i); AngelSlim documentation §2.2 (per-block budget from
// keep-ratio and alpha; sink and sliding-window blocks always kept).
// Selection: gist.science zh §2.3 (top-k key blocks per query block by the
// output-aware metric); youleyou HPC-BSA article §3.1 (the decision is taken
// outside the attention loop and handed over as a compacted list).
//
//  * budget_kernel: one CTA per sequence; budgets b_i for every query block, a
//    block-wide exclusive scan, and row_ptr for every head (the budgets do not
//    depend on the head).
//  * select_kernel: one CTA per CSR row (query head, query block).  The row's
//    causal scores are turned into order-preserving 32-bit keys (NaN -> -inf),
//    forced blocks are taken first, and an 8-bit radix select over the
//    remaining candidates finds the threshold key of the (b-|F|)-th best;
//    ties at the threshold go to the lowest indices.  Two block scans emit the
//    chosen indices in ascending order.  No host round trip; HBM-bound.
#include "stem_device.cuh"
#include "stem_kernels.h"
#include "stem_select_row.cuh"

namespace stem {

namespace {

constexpr int kSelThreads = 256;

// Inclusive block-wide scan of one int per thread (blockDim.x = kThreads).
template <int kThreads>
__device__ __forceinline__ int block_inclusive_scan(int x, int* s_warp, int* total) {
  const int lane = lane_id(), w = warp_id();
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) s_warp[w] = x;
  __syncthreads();
  if (w == 0) {
    int v = lane < kThreads / 32 ? s_warp[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, off);
      if (lane >= off) v += y;
    }
    if (lane < kThreads / 32) s_warp[lane] = v;
  }
  __syncthreads();
  const int res = x + (w > 0 ? s_warp[w - 1] : 0);
  if (total) *total = s_warp[kThreads / 32 - 1];
  __syncthreads();
  return res;
}

}  // namespace

constexpr int kBudgetThreads = 1024;

__global__ void __launch_bounds__(kBudgetThreads) budget_kernel(const SeqBatch batch, int hq, int nbtot,
                                                                 int64_t nnz_per_head, double rho, double mu,
                                                                 int sink, int window, int mode,
                                                                 int32_t* __restrict__ budgets,
                                                                 int32_t* __restrict__ row_ptr) {
  __shared__ int s_warp[32];
  const int s = blockIdx.x;
  const int nb = batch.nb[s];
  const int per = (nb + kBudgetThreads - 1) / kBudgetThreads;
  const int i0 = threadIdx.x * per;
  int local = 0;
  for (int i = i0; i < min(nb, i0 + per); ++i) local += tpd_budget(i, nb, rho, mu, sink, window, mode);
  const int incl = block_inclusive_scan<kBudgetThreads>(local, s_warp, nullptr);
  int64_t run = batch.csr0[s] + (incl - local);
  for (int i = i0; i < min(nb, i0 + per); ++i) {
    const int b = tpd_budget(i, nb, rho, mu, sink, window, mode);
    const int g = batch.g0[s] + i;
    for (int h = 0; h < hq; ++h) {
      const size_t r = static_cast<size_t>(h) * nbtot + g;
      budgets[r] = b;
      row_ptr[r] = static_cast<int32_t>(static_cast<int64_t>(h) * nnz_per_head + run);
    }
    run += b;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) row_ptr[static_cast<size_t>(hq) * nbtot] =
      static_cast<int32_t>(static_cast<int64_t>(hq) * nnz_per_head);
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(const SeqBatch batch, int h0, int nh, int group,
                                                             int nbtot, int nb_max, int sink, int window,
                                                             const float* __restrict__ scores,
                                                             const int32_t* __restrict__ budgets,
                                                             const int32_t* __restrict__ row_ptr,
                                                             int32_t* __restrict__ col_idx) {
  extern __shared__ uint32_t s_key[];  // [nb_max]
  __shared__ int s_warp[32];
  __shared__ int s_hist[256];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;

  const int s = find_seq(batch, blockIdx.x);
  const int local = blockIdx.x - batch.item0[s];
  const int nb = batch.nb[s];
  // lists of a sequence: query blocks descending (longest rows first), then
  // the lists of heads h0 .. h0 + nh - 1 (one per `group` heads)
  const int nlists = nh / group;
  const int h = h0 + (local % nlists) * group;  // first head of the list
  const int i = nb - 1 - local / nlists;
  const int g = batch.g0[s] + i;
  const size_t r = static_cast<size_t>(h) * nbtot + g;
  const int c = i + 1;
  const int b = budgets[r];
  const int nforced = static_cast<int>(forced_count(i, sink, window));
  const int ncand = c - nforced;
  const int m = min(max(b - nforced, 0), ncand);  // candidates to pick
  const float* row = scores + r * static_cast<size_t>(nb_max);
  const size_t head_stride = static_cast<size_t>(nbtot) * nb_max;  // next head's row of the same block

  // Threshold: the m-th largest candidate key (radix select, 8 bits per pass).
  uint32_t thr = 0u;
  int take_eq = 0;  // how many candidates equal to thr to take, lowest index first
  const bool all = (m == ncand);
  if (m > 0 && !all) {
    // the key of a block is that of the group's best score (order_key is
    // monotone and maps NaN below every number)
    for (int j = threadIdx.x; j < c; j += kSelThreads) {
      uint32_t k = order_key(row[j]);
      for (int e = 1; e < group; ++e) k = max(k, order_key(row[e * head_stride + j]));
      s_key[j] = k;
    }
    if (threadIdx.x == 0) {
      s_prefix = 0u;
      s_need = m;
    }
    __syncthreads();
    for (int shift = 24; shift >= 0; shift -= 8) {
      for (int q = threadIdx.x; q < 256; q += kSelThreads) s_hist[q] = 0;
      __syncthreads();
      const uint32_t pref = s_prefix;
      const uint32_t hmask = (shift == 24) ? 0u : (0xFFFFFFFFu << (shift + 8));
      for (int j = threadIdx.x; j < c; j += kSelThreads) {
        if (is_forced(j, i, sink, window)) continue;
        const uint32_t k = s_key[j];
        if ((k & hmask) == pref) atomicAdd(&s_hist[(k >> shift) & 0xFFu], 1);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        int need = s_need, acc = 0, d = 255;
        for (; d > 0; --d) {
          if (acc + s_hist[d] >= need) break;
          acc += s_hist[d];
        }
        s_need = need - acc;
        s_prefix = pref | (static_cast<uint32_t>(d) << shift);
      }
      __syncthreads();
    }
    thr = s_prefix;
    take_eq = s_need;
  }

  // Emit forced blocks, candidates above the threshold, and the first take_eq
  // candidates equal to it, in ascending index order.  Each thread owns a
  // contiguous run of indices so the scans preserve index order.
  const int per = (c + kSelThreads - 1) / kSelThreads;
  const int j0 = threadIdx.x * per;
  const int j1 = min(c, j0 + per);
  int n_eq = 0;
  if (m > 0 && !all)
    for (int j = j0; j < j1; ++j)
      if (!is_forced(j, i, sink, window) && s_key[j] == thr) ++n_eq;
  int eq_before = 0;
  if (m > 0 && !all) eq_before = block_inclusive_scan<kSelThreads>(n_eq, s_warp, nullptr) - n_eq;
  int n_sel = 0;
  {
    int e = eq_before;
    for (int j = j0; j < j1; ++j) {
      bool sel;
      if (is_forced(j, i, sink, window)) sel = true;
      else if (m <= 0) sel = false;
      else if (all) sel = true;
      else {
        const uint32_t k = s_key[j];
        sel = k > thr || (k == thr && e < take_eq);
        if (k == thr) ++e;
      }
      n_sel += sel;
    }
  }
  const int pos0 = block_inclusive_scan<kSelThreads>(n_sel, s_warp, nullptr) - n_sel;
  {
    int e = eq_before, p = pos0;
    for (int j = j0; j < j1; ++j) {
      bool sel;
      if (is_forced(j, i, sink, window)) sel = true;
      else if (m <= 0) sel = false;
      else if (all) sel = true;
      else {
        const uint32_t k = s_key[j];
        sel = k > thr || (k == thr && e < take_eq);
        if (k == thr) ++e;
      }
      if (sel) {
        for (int e = 0; e < group; ++e) col_idx[row_ptr[r + static_cast<size_t>(e) * nbtot] + p] = j;
        ++p;
      }
    }
  }
}

cudaError_t launch_budget(const SeqBatch& batch, int hq, int nbtot, int64_t nnz_per_head, double rho, double mu,
                          int sink, int window, int mode, int32_t* budgets, int32_t* row_ptr,
                          cudaStream_t stream) {
  if (batch.n == 0) return cudaSuccess;
  budget_kernel<<<batch.n, kBudgetThreads, 0, stream>>>(batch, hq, nbtot, nnz_per_head, rho, mu, sink, window,
                                                        mode, budgets, row_ptr);
  return cudaGetLastError();
}

cudaError_t launch_select(const SeqBatch& batch, int hq, int h0, int nh, int group, int nbtot, int nb_max, int sink,
                          int window, const float* scores, const int32_t* budgets, const int32_t* row_ptr,
                          int32_t* col_idx, cudaStream_t stream) {
  const int items = batch.item0[batch.n];
  if (items == 0 || nh <= 0) return cudaSuccess;
  if (h0 < 0 || h0 + nh > hq || group < 1 || nh % group != 0) return cudaErrorInvalidValue;
  const size_t smem = sizeof(uint32_t) * static_cast<size_t>(nb_max);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  select_kernel<<<items, kSelThreads, smem, stream>>>(batch, h0, nh, group, nbtot, nb_max, sink, window, scores,
                                                      budgets, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace stem
