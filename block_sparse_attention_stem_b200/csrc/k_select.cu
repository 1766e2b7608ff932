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
//  * select_kernel: one warp per list (a CSR row, or the rows of a KV group's
//    query heads that share a list).  The row's causal scores are turned into
//    order-preserving 32-bit keys (NaN -> -inf; with shared lists the best of
//    the group's scores), forced blocks are taken first, and an 8-bit radix
//    select over the remaining candidates (histograms scanned across the
//    warp) finds the threshold key of the (b-|F|)-th best; ties at the
//    threshold go to the lowest indices.  Warp scans emit the chosen indices
//    in ascending order.  No host round trip.
#include "stem_device.cuh"
#include "stem_kernels.h"
#include "stem_select_row.cuh"

namespace stem {

namespace {

constexpr int kSelWarps = 8;  // lists per CTA of the selection kernel

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

// One warp per list (warp_select_row_group); kSelWarps warps per CTA, each with
// its own keys and histogram in dynamic shared memory.
__global__ void __launch_bounds__(kSelWarps * 32) select_kernel(const SeqBatch batch, int h0, int nh, int group,
                                                                int nbtot, int nb_max, int sink, int window,
                                                                int warps_per_cta, const float* __restrict__ scores,
                                                                const int32_t* __restrict__ budgets,
                                                                const int32_t* __restrict__ row_ptr,
                                                                int32_t* __restrict__ col_idx) {
  extern __shared__ __align__(16) uint8_t s_sel[];
  const int warp = warp_id();
  const int items = batch.item0[batch.n];
  const int item = blockIdx.x * warps_per_cta + warp;
  if (warp >= warps_per_cta || item >= items) return;  // whole warps leave; nothing below syncs the CTA
  const size_t key_bytes = (static_cast<size_t>(nb_max) * 4 + 15) & ~size_t(15);
  uint32_t* keys = reinterpret_cast<uint32_t*>(s_sel + warp * (key_bytes + 1024));
  int* hist = reinterpret_cast<int*>(s_sel + warp * (key_bytes + 1024) + key_bytes);
  const int s = find_seq(batch, item);
  const int local = item - batch.item0[s];
  const int nb = batch.nb[s];
  // lists of a sequence: query blocks descending (longest rows first), then
  // the lists of heads h0 .. h0 + nh - 1 (one per `group` heads)
  const int nlists = nh / group;
  const int h = h0 + (local % nlists) * group;  // first head of the list
  const int i = nb - 1 - local / nlists;
  const size_t r = static_cast<size_t>(h) * nbtot + batch.g0[s] + i;
  warp_select_row_group(scores + r * static_cast<size_t>(nb_max), static_cast<size_t>(nbtot) * nb_max, group, i,
                        budgets[r], sink, window, keys, hist, col_idx, row_ptr, r, static_cast<size_t>(nbtot));
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
  const size_t per_warp = ((static_cast<size_t>(nb_max) * 4 + 15) & ~size_t(15)) + 1024;
  const size_t max_smem = size_t(227) << 10;
  if (per_warp > max_smem) return cudaErrorInvalidValue;
  int wpc = static_cast<int>(max_smem / per_warp);
  if (wpc > kSelWarps) wpc = kSelWarps;
  const size_t smem = per_warp * wpc;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const int grid = (items + wpc - 1) / wpc;
  select_kernel<<<grid, wpc * 32, smem, stream>>>(batch, h0, nh, group, nbtot, nb_max, sink, window, wpc, scores,
                                                  budgets, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace stem
