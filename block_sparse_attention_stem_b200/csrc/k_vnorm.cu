// k_vnorm.cu — value-magnitude bonus of the output-aware metric.
//
// "Stem" (gist.science zh summary §2.2; de summary §2 B): the metric adds
// beta * max(0, log ||V_j||^2); the value norms are max-pooled per key block.
//   vbonus[hk][g0 + j] = beta * max(0, ln max_{t in block j} ||v_t||^2)
//
// Two CTAs per key block, each taking half of the KV heads, read the block's
// 128 (or 64) tokens x Hkv heads x 128 values (256 KB bf16 in the packed
// [T, Hkv, d] layout; each CTA reads 1 KB of every 2 KB token row) once with 16-byte
// loads; 16 (bf16) or 8 (fp8) lanes cover one (token, head) row of 128
// values, and each thread keeps eight rows' loads in flight.  Measured at
// 8 KV heads (one launch each, cold L2): with four rows in flight and one CTA
// per block the pass took 65.5 us at 131072 tokens; eight rows 58.6 us, and
// two head groups 57.2 us there and 18.9 us instead of 25.7 us at 32768
// tokens, where one CTA per block leaves the SMs too few loads in flight
// (four head groups: 56.9 / 20.4 us; eight: 60.5 / 20.8 us).  The arithmetic
// per byte is small but not free (widening, packed FMAs, the row's lane
// reduction), so it is kept to a few instructions per 16-byte load.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "stem_device.cuh"
#include "stem_kernels.h"

namespace stem {

template <bool kFp8>
__global__ void __launch_bounds__(256) vnorm_kernel(const SeqBatch batch, const uint8_t* __restrict__ v,
                                                    const float* __restrict__ v_scale, int hkv, int hk_first,
                                                    int nhk_all, int heads_per_cta, int nbtot, int block,
                                                    float beta, bool raw_log, float* __restrict__ vbonus) {
  extern __shared__ unsigned int s_max[];  // [nhk] bit patterns of non-negative floats (KV heads hk0 ..)
  // this CTA's KV heads: hk0 .. hk0 + nhk - 1 (group blockIdx.y of the launch's range)
  const int hk0 = hk_first + static_cast<int>(blockIdx.y) * heads_per_cta;
  const int nhk = min(heads_per_cta, hk_first + nhk_all - hk0);
  const int s = find_seq(batch, blockIdx.x);
  const int j = blockIdx.x - batch.item0[s];
  const int t0 = j * block;
  const int ntok = min(block, batch.len[s] - t0);
  for (int h = threadIdx.x; h < nhk; h += blockDim.x) s_max[h] = 0u;
  __syncthreads();

  constexpr int kElt = kFp8 ? 1 : 2;
  constexpr int kLanesPerRow = (kHeadDim * kElt) / 16;  // 16-byte vectors per row: 16 (bf16) or 8 (fp8)
  const int rows = ntok * nhk;  // (token, head) rows of this block and head range
  const int sub = threadIdx.x % kLanesPerRow;
  const int row_step = blockDim.x / kLanesPerRow;
  const uint8_t* base = v + (static_cast<size_t>(batch.tok0[s]) + t0) * hkv * kHeadDim * kElt;
  // eight rows per thread in flight: their loads are issued before any of them
  // is reduced (the trip count is uniform across a warp, so every lane takes
  // part in the shuffles).  Row r is (token r / nhk, head r % nhk); the pair
  // is advanced by row_step without a division per row.
  constexpr int kUnroll = 8;
  const int first = threadIdx.x / kLanesPerRow;
  const int q_step = row_step / nhk, r_step = row_step % nhk;
  int quo = first / nhk, rem = first % nhk;
  for (int r0 = first; r0 - first < rows; r0 += kUnroll * row_step) {
    uint4 w[kUnroll];
    int head[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = r0 + u * row_step;
      head[u] = rem;
      w[u] = make_uint4(0u, 0u, 0u, 0u);
      if (r < rows) {
        const size_t row = static_cast<size_t>(quo) * hkv + hk0 + rem;
        w[u] = *reinterpret_cast<const uint4*>(base + row * kHeadDim * kElt + sub * 16);
      }
      quo += q_step;
      rem += r_step;
      if (rem >= nhk) {
        rem -= nhk;
        ++quo;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int r = r0 + u * row_step;
      const uint32_t q4[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
      float2 acc2 = make_float2(0.f, 0.f);  // even and odd elements, two FMAs per instruction
      if constexpr (!kFp8) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 x = make_float2(__uint_as_float(q4[q] << 16), __uint_as_float(q4[q] & 0xFFFF0000u));
          acc2 = ffma2(x, x, acc2);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
#pragma unroll
          for (int b = 0; b < 4; b += 2) {
            const __nv_fp8x2_storage_t pair = static_cast<__nv_fp8x2_storage_t>((q4[q] >> (8 * b)) & 0xFFFFu);
            const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
            const float2 x = __half22float2(*reinterpret_cast<const __half2*>(&hr));
            acc2 = ffma2(x, x, acc2);
          }
        }
      }
      float acc = acc2.x + acc2.y;
      // reduce over the lanes of this row
#pragma unroll
      for (int off = kLanesPerRow / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (r < rows && sub == 0) {
        const int h = head[u];
        if constexpr (kFp8) acc *= v_scale[hk0 + h] * v_scale[hk0 + h];
        atomicMax(&s_max[h], __float_as_uint(acc));
      }
    }
  }
  __syncthreads();
  const int g = batch.g0[s] + j;
  for (int h = threadIdx.x; h < nhk; h += blockDim.x) {
    const float m = __uint_as_float(s_max[h]);
    const float lg = logf(m);  // ln 0 = -inf -> bonus 0
    vbonus[static_cast<size_t>(hk0 + h) * nbtot + g] = raw_log ? lg : beta * fmaxf(0.f, lg);
  }
}

cudaError_t launch_vnorm(const SeqBatch& batch, const void* v, const float* v_scale, bool fp8, int hkv, int hk0,
                         int nhk, int nbtot, int block, float beta, bool raw_log, float* vbonus,
                         cudaStream_t stream) {
  const int items = batch.item0[batch.n];
  if (items == 0 || nhk <= 0) return cudaSuccess;
  const int heads_per_cta = (nhk + 1) / 2;  // two head groups (one when nhk = 1)
  const dim3 grid(items, (nhk + heads_per_cta - 1) / heads_per_cta);
  const size_t smem = sizeof(unsigned int) * static_cast<size_t>(heads_per_cta);
  if (fp8)
    vnorm_kernel<true><<<grid, 256, smem, stream>>>(batch, static_cast<const uint8_t*>(v), v_scale, hkv, hk0, nhk,
                                                    heads_per_cta, nbtot, block, beta, raw_log, vbonus);
  else
    vnorm_kernel<false><<<grid, 256, smem, stream>>>(batch, static_cast<const uint8_t*>(v), v_scale, hkv, hk0, nhk,
                                                     heads_per_cta, nbtot, block, beta, raw_log, vbonus);
  return cudaGetLastError();
}

// One CTA per (sequence, KV head): mean and population std of the finite
// x = ln max ||v||^2 over the sequence's blocks (two passes, fp64 sums), then
// bonus = beta * max(0, (x - mean) / std); 0 for a non-finite x, and for every
// block when std = 0 or no x is finite.  AngelSlim doc §2.1 (lambda *
// ReLU(v_bar), v_bar the standardized log value norm).
__global__ void __launch_bounds__(256) bonus_standardize_kernel(const SeqBatch batch, int hk0, int nbtot,
                                                                float beta, float* __restrict__ vbonus) {
  __shared__ double s_red[2][8];
  const int s = find_seq(batch, blockIdx.x);
  const int hk = hk0 + (blockIdx.x - batch.item0[s]);
  const int nb = batch.nb[s];
  float* x = vbonus + static_cast<size_t>(hk) * nbtot + batch.g0[s];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  // block-wide sum of (a, b) over the threads
  auto reduce2 = [&](double a, double b, double* ra, double* rb) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      a += __shfl_xor_sync(0xffffffffu, a, off);
      b += __shfl_xor_sync(0xffffffffu, b, off);
    }
    if (lane == 0) {
      s_red[0][w] = a;
      s_red[1][w] = b;
    }
    __syncthreads();
    double ta = 0.0, tb = 0.0;
    for (int i = 0; i < static_cast<int>(blockDim.x >> 5); ++i) {
      ta += s_red[0][i];
      tb += s_red[1][i];
    }
    __syncthreads();
    *ra = ta;
    *rb = tb;
  };
  double sum = 0.0, cnt = 0.0;
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const float v = x[j];
    if (isfinite(v)) {
      sum += v;
      cnt += 1.0;
    }
  }
  double tsum, tcnt;
  reduce2(sum, cnt, &tsum, &tcnt);
  const double mean = tcnt > 0.0 ? tsum / tcnt : 0.0;
  double sq = 0.0, unused = 0.0;
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const float v = x[j];
    if (isfinite(v)) sq += (v - mean) * (v - mean);
  }
  double tsq, tun;
  reduce2(sq, unused, &tsq, &tun);
  const double sd = tcnt > 0.0 ? sqrt(tsq / tcnt) : 0.0;
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const float v = x[j];
    const double z = (sd > 0.0 && isfinite(v)) ? (v - mean) / sd : 0.0;
    x[j] = beta * static_cast<float>(z > 0.0 ? z : 0.0);
  }
}

cudaError_t launch_bonus_standardize(const SeqBatch& batch, int hk0, int nbtot, float beta, float* vbonus,
                                     cudaStream_t stream) {
  const int items = batch.item0[batch.n];
  if (items == 0) return cudaSuccess;
  bonus_standardize_kernel<<<items, 256, 0, stream>>>(batch, hk0, nbtot, beta, vbonus);
  return cudaGetLastError();
}

}  // namespace stem
