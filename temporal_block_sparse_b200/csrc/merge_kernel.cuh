// merge_kernel.cuh -- LSE merge of partial attentions (LiteAttention README, LSE section: outputs
// over disjoint key sets, e.g. text-to-text and text-to-video for the text queries, combine into
// the attention over all keys by their log-sum-exp).
//
// For one query row with parts p = 0..P-1:
//   m = max_p lse_p,  w_p = exp(lse_p - m),  L = sum_p w_p,
//   o = sum_p (w_p / L) o_p,  lse = m + ln L.
// A part with lse_p = -inf (no key for that row) has w_p = 0; if every part is -inf the row is 0
// with lse -inf.
//
// HBM-bound: per row it reads P * (2 d + 4) bytes and writes 2 d + 4. Each thread owns 16 bytes
// (8 bf16) of one row, so a row of d = 128 is 16 consecutive threads reading whole 32-byte sectors;
// rows are walked in (b, h, n) order, which makes the lse reads of a warp contiguous too. All
// parts' loads of a thread are issued before any arithmetic, so P * 16 bytes per thread are in
// flight.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace lite {

constexpr int kMaxMergeParts = 8;

struct MergeParts {
  const __nv_bfloat16* o[kMaxMergeParts];  // [B, N, H, D] each
  const float* lse[kMaxMergeParts];        // [B, H, N] each
  int n;
};

// o / lse may alias a part's buffers (in-place merge): every thread reads all of its inputs, the
// warp (which holds whole rows) synchronises, then each thread writes only elements it has read.
// MP >= parts.n bounds the unrolled part loop (2, 4 or 8), so that few parts need few registers
// and more threads per SM keep more bytes in flight.
template <int D, int MP>
__global__ void __launch_bounds__(256) lite_lse_merge_kernel(const MergeParts parts, __nv_bfloat16* o, float* lse,
                                                             int B, int H, int N) {
  constexpr int G = D / 8;  // threads per row
  const long long rows = static_cast<long long>(B) * H * N;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  // the loop bound is uniform over a warp (whole warps step together), so __syncwarp is legal
  const long long warp_base0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) & ~31ll;
  const int lane = threadIdx.x & 31;
  for (long long base = warp_base0; base < rows * G; base += stride) {
    const long long gid = base + lane;
    const bool valid = gid < rows * G;
    const long long row = valid ? gid / G : 0;  // (b * H + h) * N + n
    const int g = int(gid - row * G);
    const long long bh = row / N;
    const int n = int(row - bh * N);
    const int b = int(bh / H);
    const int h = int(bh - static_cast<long long>(b) * H);
    const size_t off = ((static_cast<size_t>(b) * N + n) * H + h) * D + size_t(g) * 8;

    float l[MP];
    uint4 v[MP];
#pragma unroll
    for (int p = 0; p < MP; ++p) {
      if (p < parts.n && valid) {
        l[p] = parts.lse[p][row];
        v[p] = *reinterpret_cast<const uint4*>(parts.o[p] + off);
      } else {
        l[p] = -INFINITY;
        v[p] = make_uint4(0, 0, 0, 0);
      }
    }
    __syncwarp();
    float m = -INFINITY;
#pragma unroll
    for (int p = 0; p < MP; ++p) m = fmaxf(m, l[p]);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float out_lse = -INFINITY;
    if (m > -INFINITY) {
      float w[MP];
      float tot = 0.f;
#pragma unroll
      for (int p = 0; p < MP; ++p) {
        w[p] = (l[p] > -INFINITY) ? expf(l[p] - m) : 0.f;
        tot += w[p];
      }
      const float inv = 1.f / tot;
#pragma unroll
      for (int p = 0; p < MP; ++p) {
        if (w[p] == 0.f) continue;
        const float wp = w[p] * inv;
        const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&v[p]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(x[e]);
          acc[2 * e] = fmaf(wp, f.x, acc[2 * e]);
          acc[2 * e + 1] = fmaf(wp, f.y, acc[2 * e + 1]);
        }
      }
      out_lse = m + logf(tot);
    }
    if (valid) {
      uint4 res;
      uint32_t* r = reinterpret_cast<uint32_t*>(&res);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
        r[e] = *reinterpret_cast<uint32_t*>(&h2);
      }
      *reinterpret_cast<uint4*>(o + off) = res;
      if (lse && g == 0) lse[row] = out_lse;
    }
  }
}

}  // namespace lite
