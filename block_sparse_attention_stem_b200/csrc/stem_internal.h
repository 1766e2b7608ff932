// stem_internal.h — definitions shared by the host side of the library and
// its kernels: launch-batch descriptors, the position-decay budget (one
// function compiled for both host and device so the planner's nnz and the
// device's budgets are the same numbers), and the workspace layout.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define STEM_HD __host__ __device__ __forceinline__
#else
#define STEM_HD inline
#endif

namespace stem {

// Must equal the stem_status_t values of include/stem.h.
constexpr int STEM_ERR_TIMEOUT_CODE = 6;
constexpr int STEM_ERR_BAD_BLOCKLIST_CODE = 7;

constexpr int kBlock = 128;      // block (tokens); also the attention's query tile for 64-token blocks
constexpr int kMaxBitmapBlocks = 32768;  // 64-token blocks: longest sequence in blocks (2,097,152 tokens)
constexpr int kHeadDim = 128;    // supported head_dim
constexpr int kMaxSeqPerLaunch = 8;

// Sequences handled by one kernel launch.  Work items of sequence s are
// item0[s] .. item0[s+1]-1.
struct SeqBatch {
  int32_t n;                          // sequences in this launch
  int32_t tok0[kMaxSeqPerLaunch];     // first packed token of the sequence
  int32_t len[kMaxSeqPerLaunch];      // L_s
  int32_t nb[kMaxSeqPerLaunch];       // NB_s = ceil(L_s / 128)
  int32_t g0[kMaxSeqPerLaunch];       // global index of the sequence's block 0
  int32_t item0[kMaxSeqPerLaunch + 1];
  int64_t csr0[kMaxSeqPerLaunch];     // CSR offset of the sequence's first row inside one head
  int32_t seq_id[kMaxSeqPerLaunch];   // the sequence's number in the call (cu_seqlens order)
};

STEM_HD int find_seq(const SeqBatch& b, int item) {
  int s = 0;
  while (s + 1 < b.n && item >= b.item0[s + 1]) ++s;
  return s;
}

// IEEE fp64 round-to-nearest arithmetic without contraction, identical on
// host (SSE2, -ffp-contract=off) and device (explicit _rn intrinsics).
STEM_HD double d_mul(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dmul_rn(a, b);
#else
  return a * b;
#endif
}
STEM_HD double d_sub(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dsub_rn(a, b);
#else
  return a - b;
#endif
}
STEM_HD double d_div(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __ddiv_rn(a, b);
#else
  return a / b;
#endif
}
STEM_HD double d_floor(double x) {
#if defined(__CUDA_ARCH__)
  return floor(x);
#else
  return __builtin_floor(x);
#endif
}
STEM_HD double d_ceil(double x) {
#if defined(__CUDA_ARCH__)
  return ceil(x);
#else
  return __builtin_ceil(x);
#endif
}

STEM_HD int64_t i64min(int64_t a, int64_t b) { return a < b ? a : b; }
STEM_HD int64_t i64max(int64_t a, int64_t b) { return a > b ? a : b; }

// |F_i| for F_i = {0 .. min(S,c)-1} u {max(0,c-W) .. c-1}, c = i + 1.
STEM_HD int64_t forced_count(int64_t i, int64_t sink, int64_t window) {
  const int64_t c = i + 1;
  const int64_t a = i64min(sink, c);
  const int64_t bs = i64max(int64_t(0), c - window);
  return a + (c - bs) - i64max(int64_t(0), a - bs);
}

STEM_HD bool is_forced(int64_t j, int64_t i, int64_t sink, int64_t window) {
  const int64_t c = i + 1;
  return j < i64min(sink, c) || j >= c - window;
}

// Token position-decay budget of query block i in a sequence of nb blocks
// ("Stem", gist.science zh summary §2.1: k(i) = floor(k_start -
// k_start (1 - mu) / N * i)); keep-ratio mapping RELATIVE (mode 0:
// k_start = ceil(rho (i+1))) or ABSOLUTE (mode 1: ceil(rho nb)); forced
// sink/window blocks count inside the budget, capped by the i+1 causal blocks.
STEM_HD int32_t tpd_budget(int64_t i, int64_t nb, double rho, double mu, int64_t sink, int64_t window,
                           int mode) {
  const int64_t c = i + 1;
  const double base = (mode == 0) ? static_cast<double>(c) : static_cast<double>(nb);
  const double ks = d_ceil(d_mul(rho, base));
  const double t = d_div(d_mul(d_mul(ks, d_sub(1.0, mu)), static_cast<double>(i)), static_cast<double>(nb));
  const int64_t k = static_cast<int64_t>(d_floor(d_sub(ks, t)));
  const int64_t nf = forced_count(i, sink, window);
  return static_cast<int32_t>(i64min(c, i64max(k, nf)));
}

}  // namespace stem
