// calib_kernels.cuh -- dropped softmax mass of a Skip-Mask, for the accumulated-error calibration of
// the QK-Skip threshold ("Lite Attention Temporal Sparse" skill page, Architecture Overview:
// Accumulated-Error Calibration; LiteAttention README, "Error Calibration").
//
// For every query row, the probability mass that the skipped key tiles hold under the dense softmax
// is 1 - Z_live / Z_full = -expm1(lse_live - lse_full), with lse_live the log-normaliser over the
// live tiles only (lite_attn_fwd with the mask as input) and lse_full the dense one
// (lite_attn_dense). A row with no live tile (lse_live = -inf) drops everything (1).
//
// HBM-bound: 8 bytes read per row (+4 written when the per-row values are requested). Grid-stride
// loop with 4 rows per thread (16-byte loads), block reduction of the maximum and the sum through
// warp shuffles, one atomic of each per block into stats[2] = {max, sum} (zeroed by the host).
#pragma once

#include <stdint.h>

namespace lite {

__device__ __forceinline__ float dropped_one(float live, float full) {
  if (live == -INFINITY) return 1.f;
  const float m = -expm1f(live - full);
  return fminf(fmaxf(m, 0.f), 1.f);
}

__global__ void __launch_bounds__(256) lite_dropped_mass_kernel(const float* __restrict__ lse_live,
                                                                const float* __restrict__ lse_full,
                                                                float* __restrict__ row_mass, float* stats,
                                                                long long rows) {
  float mx = 0.f, sum = 0.f;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x * 4;
  const bool vec = ((reinterpret_cast<uintptr_t>(lse_live) | reinterpret_cast<uintptr_t>(lse_full) |
                     reinterpret_cast<uintptr_t>(row_mass)) & 15u) == 0;
  for (long long base = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 4; base < rows;
       base += stride) {
    float m[4];
    if (vec && base + 4 <= rows) {
      const float4 a = *reinterpret_cast<const float4*>(lse_live + base);
      const float4 f = *reinterpret_cast<const float4*>(lse_full + base);
      m[0] = dropped_one(a.x, f.x);
      m[1] = dropped_one(a.y, f.y);
      m[2] = dropped_one(a.z, f.z);
      m[3] = dropped_one(a.w, f.w);
      if (row_mass) *reinterpret_cast<float4*>(row_mass + base) = make_float4(m[0], m[1], m[2], m[3]);
    } else {
      for (int e = 0; e < 4; ++e) {
        m[e] = base + e < rows ? dropped_one(lse_live[base + e], lse_full[base + e]) : 0.f;
        if (row_mass && base + e < rows) row_mass[base + e] = m[e];
      }
    }
    mx = fmaxf(mx, fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])));
    sum += (m[0] + m[1]) + (m[2] + m[3]);
  }
  for (int o = 16; o > 0; o >>= 1) {
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    sum += __shfl_xor_sync(0xffffffffu, sum, o);
  }
  __shared__ float smx[8], ssum[8];
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    smx[w] = mx;
    ssum[w] = sum;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = 0.f, bs = 0.f;
    for (int i = 0; i < int(blockDim.x >> 5); ++i) {
      bm = fmaxf(bm, smx[i]);
      bs += ssum[i];
    }
    // the values are in [0, 1]: their IEEE bit patterns order like the values
    atomicMax(reinterpret_cast<unsigned int*>(stats), __float_as_uint(bm));
    atomicAdd(stats + 1, bs);
  }
}

}  // namespace lite
