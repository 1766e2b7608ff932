// k_vwiden.cu — V widened from e4m3 to f16 for the fp8 attention path.
//
// The fp8 attention kernel keeps P in f16 (an e4m3 P would carry three
// mantissa bits) and runs P V as an f16 product, so V is widened once per call.
// Every e4m3 value is an f16 value, so the widening is exact; the dequantisation
// scale stays separate (the kernel applies it to O).  youleyou HPC-BSA article
// §3.1 (fp8 K/V storage, block-sparse prefill); AngelSlim documentation §5 (the
// paged fp8 KV path), whose page-table lookup this pass also performs, so that
// the attention kernel reads V packed.
//
// HBM-bound: each 128-dim row is 128 bytes in and 256 bytes out; every thread
// moves one 16-byte unit (16 values) per iteration of a grid-stride loop.
#include "stem_device.cuh"
#include "stem_kernels.h"

namespace stem {

namespace {

constexpr int kWidenThreads = 256;

__device__ __forceinline__ uint32_t widen2(uint32_t word, int pair) {
  return e4m3x2_to_f16x2(static_cast<uint16_t>(word >> (16 * pair)));
}

}  // namespace

// Output row (t, hk) for tokens t < total_tokens and KV heads hk0 .. hk0+nhk-1:
// the packed input row (t, hk), or, with a page table, row u % page_size of
// page page_table[s][u / page_size] (s the sequence of t, u = t - cu_seqlens[s]);
// a page number outside [0, num_pages) gives zeros.
__global__ void __launch_bounds__(kWidenThreads)
    vwiden_kernel(const uint8_t* __restrict__ v8, uint16_t* __restrict__ v16, int total_tokens, int hkv, int hk0,
                  int nhk, const int32_t* __restrict__ cu_seqlens, int num_seqs,
                  const int32_t* __restrict__ page_table, int page_size, int num_pages, int max_pages) {
  const int64_t units = static_cast<int64_t>(total_tokens) * nhk * 8;  // 8 units of 16 values per row
  for (int64_t u = static_cast<int64_t>(blockIdx.x) * kWidenThreads + threadIdx.x; u < units;
       u += static_cast<int64_t>(gridDim.x) * kWidenThreads) {
    const int part = static_cast<int>(u & 7);
    const int64_t rowi = u >> 3;
    const int hk = hk0 + static_cast<int>(rowi % nhk);
    const int64_t t = rowi / nhk;
    int64_t src = t;
    bool zero = false;
    if (page_table != nullptr) {
      // the sequence of t: the last s with cu_seqlens[s] <= t
      int lo = 0, hi = num_seqs - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(cu_seqlens + mid) <= t) lo = mid;
        else hi = mid - 1;
      }
      const int64_t local = t - __ldg(cu_seqlens + lo);
      const int pg = __ldg(page_table + static_cast<size_t>(lo) * max_pages + local / page_size);
      zero = pg < 0 || pg >= num_pages;
      src = static_cast<int64_t>(pg) * page_size + local % page_size;
    }
    uint4 in = make_uint4(0u, 0u, 0u, 0u);
    if (!zero) in = __ldg(reinterpret_cast<const uint4*>(v8 + (static_cast<size_t>(src) * hkv + hk) * kHeadDim) + part);
    uint4* dst = reinterpret_cast<uint4*>(v16 + (static_cast<size_t>(t) * hkv + hk) * kHeadDim) + 2 * part;
    dst[0] = make_uint4(widen2(in.x, 0), widen2(in.x, 1), widen2(in.y, 0), widen2(in.y, 1));
    dst[1] = make_uint4(widen2(in.z, 0), widen2(in.z, 1), widen2(in.w, 0), widen2(in.w, 1));
  }
}

cudaError_t launch_vwiden(const void* v8, uint16_t* v16, int total_tokens, int hkv, int hk0, int nhk,
                          const int32_t* cu_seqlens, int num_seqs, const int32_t* page_table, int page_size,
                          int num_pages, int max_pages, cudaStream_t stream) {
  if (total_tokens <= 0 || nhk <= 0) return cudaSuccess;
  if (hk0 < 0 || hk0 + nhk > hkv) return cudaErrorInvalidValue;
  int sms = 0, dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const int64_t units = static_cast<int64_t>(total_tokens) * nhk * 8;
  const int64_t want = (units + kWidenThreads - 1) / kWidenThreads;
  const int grid = static_cast<int>(want < static_cast<int64_t>(sms) * 8 ? want : static_cast<int64_t>(sms) * 8);
  vwiden_kernel<<<grid, kWidenThreads, 0, stream>>>(static_cast<const uint8_t*>(v8), v16, total_tokens, hkv, hk0,
                                                    nhk, cu_seqlens, num_seqs, page_table, page_size, num_pages,
                                                    max_pages);
  return cudaGetLastError();
}

}  // namespace stem
