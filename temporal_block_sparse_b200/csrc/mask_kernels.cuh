// mask_kernels.cuh -- Skip-Mask bookkeeping on the device.
//
//  * lite_compact_kernel: Skip-Mask -> Skip-List. One warp per (b, h, query tile). The mask row is
//    read one 32-bit word at a time from the top word down; lane l owns key tile 32*w + 31 - l, so a
//    ballot plus a prefix popcount gives every live tile its slot in descending order (the README's
//    reverse iteration order). The same pass copies the row into mask_out (with bits >= T cleared),
//    which is where the attention kernel later ORs new flags. With must-do / must-skip ranges the
//    live set is (not masked or must-do) and not (must-skip and not must-do); must-do entries are
//    tagged so that the attention kernel never flags them. The copied mask is mask_in unchanged.
//  * lite_stride_score_kernel: for each candidate pairing stride s, the number of live key tiles
//    the attention kernel's query-tile pairs would share (summed over heads). A key tile live for
//    both query tiles of a pair is loaded once and computed for both with their softmaxes
//    overlapping; one live for only one of them runs alone. Pairing the tiles that share the most
//    live key tiles therefore cuts such lone tiles: on the 720p-like layers the best stride is 28,
//    the tiles one latent frame apart (3600 tokens per frame / 128).
//  * lite_schedule_kernel: one CTA per head. Ranks the head among all heads by total live work,
//    then places each of its work items (query tiles, or pairs of query tiles) by (live count
//    desc, index asc) with an O(T^2) rank count in shared memory -- deterministic, no atomics on
//    the output. For pairs it first picks the stride with the best score (ties: the smaller).
#pragma once

#include <stdint.h>

#include "attn_kernel.cuh"

namespace lite {

// Key tiles pinned by must-do / must-skip token ranges (README, must_do_list / must_skip_list),
// as bitmaps in the Skip-Mask's word layout. Passed by value: Tk <= 4096 gives at most 128 words.
struct RangeBits {
  uint32_t live[128];  // must-do: always live, never flagged
  uint32_t skip[128];  // must-skip (must-do already removed): always skipped
};

// Words of one mask row into registers: lane l gets words l, l + 32, l + 64, l + 96 (0 past W;
// bits >= T of the last word cleared). Rows have at most 128 words (T <= 4096).
__device__ __forceinline__ void load_row_words(const uint32_t* mask, size_t row, int W, int T, int lane,
                                               uint32_t (&wr)[4]) {
  const uint32_t tail_mask = (T & 31) ? ((1u << (T & 31)) - 1u) : 0xffffffffu;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int w = lane + 32 * i;
    uint32_t v = 0u;
    if (w < W) {
      v = mask ? mask[row * W + w] : 0u;
      if (w == W - 1) v &= tail_mask;
    }
    wr[i] = v;
  }
}

// Word w of the row, broadcast to the whole warp (w is warp-uniform).
__device__ __forceinline__ uint32_t row_word(const uint32_t (&wr)[4], int w) {
  const int i = w >> 5;
  const uint32_t mine = i == 0 ? wr[0] : (i == 1 ? wr[1] : (i == 2 ? wr[2] : wr[3]));
  return __shfl_sync(0xffffffffu, mine, w & 31);
}

// mask_in may alias mask_out (in-place update): each warp reads its row before it writes it back.
// kRanges: apply RangeBits (live wins over skip and over the mask; tagged entries are never flagged).
template <bool kRanges>
__global__ void __launch_bounds__(256) lite_compact_kernel(const uint32_t* mask_in, uint32_t* mask_out,
                                                          int16_t* __restrict__ list, int32_t* __restrict__ counts,
                                                          int rows, int T, int W, const RangeBits ranges) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_global >= rows) return;
  const size_t row = size_t(warp_global);
  // The row's words are read in one round (lane l holds words l, l+32, l+64, l+96; W <= 128), so
  // the warp waits for memory once, not once per word; the copy to mask_out is written the same
  // way. In place (mask_out == mask_in) is safe: every word of the row is read before any write.
  uint32_t wr[4];
  load_row_words(mask_in, row, W, T, lane, wr);
  if (mask_out) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (lane + 32 * i < W) mask_out[row * W + lane + 32 * i] = wr[i];
  }
  int count = 0;
  for (int w = W - 1; w >= 0; --w) {
    uint32_t word = row_word(wr, w);
    uint32_t forced = 0u;
    if constexpr (kRanges) {
      forced = ranges.live[w];
      word = (word | ranges.skip[w]) & ~forced;
    }
    const int j = w * 32 + 31 - lane;
    const bool live = (j < T) && !((word >> (31 - lane)) & 1u);
    const uint32_t bal = __ballot_sync(0xffffffffu, live);
    if (live && list) {
      const int tag = ((forced >> (31 - lane)) & 1u) ? kListNoFlag : 0;
      list[row * T + count + __popc(bal & ((1u << lane) - 1u))] = int16_t(j | tag);
    }
    count += __popc(bal);
  }
  if (lane == 0) counts[row] = count;
}

// Skip-Mask -> range-encoded Skip-List ("Lite Attention Temporal Sparse" skill page, Architecture
// Overview: the skip state is a bitmask, or a list where sparsity is high; README must_do_list
// convention for ranges: pairs (start inclusive, end exclusive) in strictly descending order,
// walked from the top down).
// A run of live key tiles a..b (a <= b) becomes the pair (b, a - 1). One warp per (b, h, query
// tile), words from the top down, lane l owns key tile 32w + 31 - l. A live tile opens a run when
// the tile above it is not live and closes one when the tile below is not live; ballots of both
// flags and their prefix popcounts place each lane's start / end entries in order. The tile above
// lane 0 is the previous word's lane 31 (carried); the tile below lane 31 is bit 31 of the next
// lower word (read ahead).
__global__ void __launch_bounds__(256) lite_ranges_kernel(const uint32_t* __restrict__ mask, int16_t* __restrict__ ranges,
                                                         int32_t* __restrict__ nruns, int rows, int T, int W) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_global >= rows) return;
  const size_t row = size_t(warp_global);
  const int R = T + 1;  // entries per row: at most 2 * ceil(T / 2) <= T + 1
  const uint32_t tail_mask = (T & 31) ? ((1u << (T & 31)) - 1u) : 0xffffffffu;
  const uint32_t below_me = (1u << lane) - 1u;  // lanes with a higher tile index
  uint32_t wr[4];
  load_row_words(mask, row, W, T, lane, wr);   // one round of loads for the whole row
  auto live_bits = [&](int w) -> uint32_t {     // bit i set = tile 32w + i live
    const uint32_t valid = (w == W - 1) ? tail_mask : 0xffffffffu;
    return ~row_word(wr, w) & valid;
  };
  int count = 0;
  bool above_live = false;  // tile 32(w+1) (lane 31 of the word above)
  uint32_t cur = live_bits(W - 1);
  for (int w = W - 1; w >= 0; --w) {
    const uint32_t next = w > 0 ? live_bits(w - 1) : 0u;
    const int j = w * 32 + 31 - lane;
    const bool live = (cur >> (31 - lane)) & 1u;
    const bool up = lane == 0 ? above_live : ((cur >> (32 - lane)) & 1u);      // tile j + 1
    const bool down = lane == 31 ? ((next >> 31) & 1u) : ((cur >> (30 - lane)) & 1u);  // tile j - 1
    const bool start = live && !up;
    const bool end = live && !down;
    const uint32_t bs = __ballot_sync(0xffffffffu, start);
    const uint32_t be = __ballot_sync(0xffffffffu, end);
    const int off = count + __popc(bs & below_me) + __popc(be & below_me);
    if (start) ranges[row * R + off] = int16_t(j);
    if (end) ranges[row * R + off + (start ? 1 : 0)] = int16_t(j - 1);
    count += __popc(bs) + __popc(be);
    above_live = cur & 1u;
    cur = next;
  }
  if (lane == 0) nruns[row] = count / 2;
}

constexpr int kMaxPairStride = 64;

// Candidate stride s = blockIdx.x + 1; blockIdx.y splits the heads. scores[s-1] (zeroed before the
// launch) += live key tiles shared by the pairs of stride s, over this block's heads. Every mask row
// is read whole (bits >= Tk of the last word cleared).
__global__ void __launch_bounds__(256) lite_stride_score_kernel(const uint32_t* __restrict__ mask,
                                                               uint32_t* __restrict__ scores, int BH, int T, int Tk,
                                                               int W) {
  const int s = blockIdx.x + 1;
  const int P = (T + 1) / 2;  // T: query tiles per head; Tk: key tiles (bits per row)
  const uint32_t tail_mask = (Tk & 31) ? ((1u << (Tk & 31)) - 1u) : 0xffffffffu;
  const long long items = static_cast<long long>(BH) * P;
  const long long per = (items + gridDim.y - 1) / gridDim.y;
  const long long lo = per * blockIdx.y, hi = min(items, lo + per);
  uint32_t acc = 0;
  for (long long x = lo + threadIdx.x; x < hi; x += blockDim.x) {
    const int bh = int(x / P);
    const int k = int(x - static_cast<long long>(bh) * P);
    int a, b;
    pair_tiles(k, T, s, a, b);
    if (b < 0) continue;
    const uint32_t* ra = mask + (size_t(bh) * T + a) * W;
    const uint32_t* rb = mask + (size_t(bh) * T + b) * W;
    for (int w = 0; w < W; ++w) {
      const uint32_t valid = (w == W - 1) ? tail_mask : 0xffffffffu;
      acc += __popc(~__ldg(ra + w) & ~__ldg(rb + w) & valid);
    }
  }
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint32_t part[8];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
    for (int i = 0; i < int(blockDim.x >> 5); ++i) t += part[i];
    if (t) atomicAdd(scores + (s - 1), t);
  }
}

// The pairing stride for G = 2: fixed_stride if >= 1, else the candidate with the highest score
// (the smaller stride on ties), 1 without scores.
__device__ __forceinline__ int pick_stride(const uint32_t* scores, int n_cand, int fixed_stride) {
  if (fixed_stride >= 1) return fixed_stride;
  if (!scores) return 1;
  int best = 1;
  uint32_t top = scores[0];
  for (int x = 1; x < n_cand; ++x)
    if (scores[x] > top) {
      top = scores[x];
      best = x + 1;
    }
  return best;
}

// smem: totals[BH] ints, then counts of this head [T] ints
// G = 1 orders the query tiles of every head; G = 2 orders pairs of query tiles (pair_tiles with the
// picked stride, which CTA 0 also writes to *stride_out), the work items of the attention kernel, by
// their combined live count; G = 4 orders the work items of the stacked-row attention kernel (d = 64:
// a pair of 128-row kernel query tiles, each two mask rows), by the live count of their four mask
// rows, consecutive kernel tiles assumed (the stride written is the option's, else 1). Output
// entries are head * ceil(T/G) + item.
template <int G>
__global__ void __launch_bounds__(512) lite_schedule_kernel(const int32_t* __restrict__ counts,
                                                           int32_t* __restrict__ order, int BH, int T,
                                                           const uint32_t* scores = nullptr, int n_cand = 0,
                                                           int fixed_stride = 0, int* stride_out = nullptr) {
  extern __shared__ int32_t sh[];
  const int P = (T + G - 1) / G;  // items per head
  int32_t* totals = sh;
  int32_t* mine = sh + BH;
  const int g = blockIdx.x;
  const int stride = G >= 2 ? pick_stride(scores, n_cand, fixed_stride) : 1;
  if (G >= 2 && g == 0 && threadIdx.x == 0 && stride_out) *stride_out = stride;
  for (int x = threadIdx.x; x < BH; x += blockDim.x) totals[x] = 0;
  __syncthreads();
  // per-head totals (every CTA computes all of them; B*H*T ints, served from L2)
  for (int x = threadIdx.x; x < BH * T; x += blockDim.x) {
    const int v = __ldg(counts + x);
    if (v) atomicAdd(&totals[x / T], v);
  }
  for (int x = threadIdx.x; x < P; x += blockDim.x) {
    int c = 0;
    if constexpr (G == 2) {
      int a, b;
      pair_tiles(x, T, stride, a, b);
      c = __ldg(counts + size_t(g) * T + a) + (b >= 0 ? __ldg(counts + size_t(g) * T + b) : 0);
    } else {
#pragma unroll
      for (int k = 0; k < G; ++k)
        if (G * x + k < T) c += __ldg(counts + size_t(g) * T + G * x + k);
    }
    mine[x] = c;
  }
  __syncthreads();
  // rank of this head: heads with more work, or equal work and a lower index, go first
  const int my_total = totals[g];
  __shared__ int rank_acc;
  if (threadIdx.x == 0) rank_acc = 0;
  __syncthreads();
  int before = 0;
  for (int x = threadIdx.x; x < BH; x += blockDim.x)
    before += (totals[x] > my_total) || (totals[x] == my_total && x < g);
  atomicAdd(&rank_acc, before);
  __syncthreads();
  const size_t base = size_t(rank_acc) * P;
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    const int c = mine[i];
    int pos = 0;
    for (int x = 0; x < P; ++x) {
      const int cx = mine[x];
      pos += (cx > c) || (cx == c && x < i);
    }
    order[base + pos] = g * P + i;
  }
}

}  // namespace lite
