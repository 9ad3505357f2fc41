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
// HBM-bound: per row it reads P * (2 d + 4) bytes and writes 2 d + 4. A thread owns 16-byte pieces
// (8 bf16) of rows: with two parts, two pieces a grid stride apart per iteration, whose loads are
// all issued before any arithmetic (64 bytes in flight per thread; more pieces cost more than they
// gain). Rows are walked in memory order of o, (b, n, h), so a warp reads and writes one contiguous
// 512-byte stretch of every part (d = 128: two rows); the lse values it needs are strided by N but
// few (24 MB for a 720p layer's two parts), and the n-neighbours that share their sectors are
// processed right after, out of L2. Index arithmetic is 32-bit (the host refuses
// B*H*N*d/8 >= 2^31).
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
__device__ __forceinline__ void merge_one(const MergeParts& parts, const float (&l)[MP], const uint4 (&v)[MP],
                                          __nv_bfloat16* o, float* lse, size_t off, size_t lrow, bool write_lse) {
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
  uint4 res;
  uint32_t* r = reinterpret_cast<uint32_t*>(&res);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
    r[e] = *reinterpret_cast<uint32_t*>(&h2);
  }
  *reinterpret_cast<uint4*>(o + off) = res;
  if (lse && write_lse) lse[lrow] = out_lse;
}

// o / lse may alias a part's buffers (in-place merge): every thread reads all of its inputs, the
// warp (which holds whole rows) synchronises, then each thread writes only elements it has read.
// MP >= parts.n bounds the unrolled part loop (2, 4 or 8), so that few parts need few registers.
// Each thread takes U 16-byte pieces a grid stride apart per iteration and issues all their loads
// before any arithmetic, so U * parts * 16 bytes are in flight per thread.
template <int D, int MP>
__global__ void __launch_bounds__(256) lite_lse_merge_kernel(const MergeParts parts, __nv_bfloat16* o, float* lse,
                                                             int B, int H, int N) {
  constexpr int G = D / 8;  // threads per row
  constexpr int U = MP <= 2 ? 2 : 1;
  const uint32_t total = uint32_t(B) * H * N * G;
  const uint32_t stride = gridDim.x * blockDim.x;
  // the loop bound is uniform over a warp (whole warps step together), so __syncwarp is legal
  const uint32_t warp_base0 = (blockIdx.x * blockDim.x + threadIdx.x) & ~31u;
  const uint32_t lane = threadIdx.x & 31;
  for (uint32_t base = warp_base0; base < total; base += U * stride) {
    float l[U][MP];
    uint4 v[U][MP];
    size_t off[U], lrow[U];
    bool valid[U], lead[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t gid = base + u * stride + lane;
      valid[u] = gid < total;
      const uint32_t row = valid[u] ? gid / G : 0;  // (b * N + n) * H + h: the memory order of o
      const uint32_t g = gid - row * G;
      const uint32_t bn = row / uint32_t(H);
      const uint32_t h = row - bn * uint32_t(H);
      const uint32_t b = bn / uint32_t(N);
      const uint32_t n = bn - b * uint32_t(N);
      off[u] = size_t(row) * D + g * 8;
      lrow[u] = (size_t(b) * H + h) * N + n;
      lead[u] = g == 0;
#pragma unroll
      for (int p = 0; p < MP; ++p) {
        if (p < parts.n && valid[u]) {
          l[u][p] = parts.lse[p][lrow[u]];
          v[u][p] = *reinterpret_cast<const uint4*>(parts.o[p] + off[u]);
        } else {
          l[u][p] = -INFINITY;
          v[u][p] = make_uint4(0, 0, 0, 0);
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (valid[u]) merge_one<D, MP>(parts, l[u], v[u], o, lse, off[u], lrow[u], lead[u]);
  }
}

}  // namespace lite
