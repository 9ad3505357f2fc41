// attn_kernel.cuh -- persistent block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// Persistent CTAs (one per SM with d = 128; two per SM with d = 64, whose CTA needs half the TMEM
// columns) walk a list of work items; an item is a pair of 128-row query tiles of one
// (b, h): tile r and tile r + s of each block of 2s tiles, with the pairing stride s chosen per call
// as the one whose pairs share the most live key tiles (s = 28 on 720p-like layers, one latent frame
// apart). With d = 64 a 128-row query tile stacks two 64-row Skip-Mask rows, each with its own list.
// For each query tile it computes only the live key tiles of that tile (LiteAttention README,
// "Full-Stage Elimination": a skipped tile costs no K/V load, no QK^T, no softmax, no PV), from the
// highest key-tile index down (README, must_do_list: the kernel walks key tiles in reverse
// order). The two query tiles share K/V: the CTA walks the union of their Skip-Lists, loads each
// union tile once, and computes it for the query tiles it is live for. Queries and keys may differ
// in length (README, LSE section: partial attentions such as text-to-video over a subset of the
// keys); a key tile that a must-do range keeps live carries a tag in its list entry and is computed
// but never flagged.
//
// Warp roles (320 threads):
//   warp 0       TMA producer: per item the pair's two Q tiles; per union tile u a load bundle with
//                K_u (2-stage ring) and V_{u-1} (2-stage ring), one barrier per bundle. It walks the
//                two lists, checks them (in range, strictly descending; a bad list, live count or
//                work-order entry stops the kernel with LITE_ERR_CHECK in the status word), and
//                hands the MMA thread, per union tile, which query tiles it is live for, in a small
//                shared-memory ring written before the bundle is armed.
//   warp 1       TMEM allocator and single-thread tcgen05 MMA issuer. Per union tile u, for query
//                tile g = 0, 1: PV_g(u-1) if u-1 was live for g, then QK_g(u) if u is live for g:
//                  S_g = Q_g K_u^T    (SS form) into TMEM buffer g,
//                  O_g += P_g V_{u-1} (TS form: P read from TMEM, V from shared memory).
//   warps 2..5   softmax warpgroup 0, query tile 0 of the pair; warps 6..9: group 1, query tile 1.
//                One thread per query row (TMEM lane). Per live tile of its query tile: row max;
//                the QK-Skip vote (skill page "Lite Attention Temporal Sparse", Core Concept: a
//                tile whose local max score is far below the cumulative max is flagged) against
//                the running max over the tile's earlier live tiles; one atomicOr per flagged
//                (query tile, key tile); exp2 (a sixteenth on the FMA pipe); P (bf16) back into TMEM
//                over the consumed S columns; O rescale when the reference max grew by more than
//                kRescaleLog2. The two groups run on the two query tiles at once, so the latency of
//                one hides the other's.
//
// Every wait is bounded by a wall-clock limit; on expiry the kernel records a timeout in the device
// status word, every role stops, in-flight copies and MMAs are drained, TMEM is freed and the CTA
// exits. No trap, no unbounded spin.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "sm100_ptx.cuh"

namespace lite {

constexpr int kStatusTimeout = -4;  // LITE_ERR_TIMEOUT
constexpr int kStatusCheck = -5;    // LITE_ERR_CHECK

// Skip-List entries are key-tile indices (< 4096). Bit 14 marks a tile that a must-do range keeps
// live: it is computed like any other tile but never flagged.
constexpr int kListIndexMask = 0x0fff;
constexpr int kListNoFlag = 0x4000;

struct AttnParams {
  __nv_bfloat16* o;         // [B, Nq, H, D]
  float* lse;               // [B, H, Nq] or null
  uint32_t* mask_out;       // [B, H, Tq, W] or null (flags not recorded)
  const int16_t* list;      // [B*H*Tq, Tk] live key tiles, descending (null: all tiles, dense)
  const int32_t* counts;    // [B*H*Tq] live counts (null: Tk each)
  const int32_t* order;     // [n_items] work order over query-tile pairs (null: identity)
  int32_t* work_counter;    // zero before launch; null = static striding over items
  int* status;              // device status word
  int B, H;
  int Nq, Nk;               // query / key tokens (equal for self attention)
  int Tq, Tk, W;            // query tiles (mask rows), key tiles, mask words per row (ceil(Tk / 32))
  int Tkq;                  // kernel query tiles per (b, h): ceil(Tq / MR)
  int Pq;                   // work items (kernel query-tile pairs) per (b, h): ceil(Tkq / 2)
  int n_items;              // B * H * Pq
  const int* pair_stride_ptr;  // pairing stride chosen on the device for this call (null: pair_stride)
  int pair_stride;             // pairing stride when pair_stride_ptr is null (1: tiles 2k and 2k+1)
  float scale_log2;         // softmax scale * log2(e)
  float tau_log2;           // QK-Skip threshold * log2(e)
  int skip_test;            // 1: run the QK-Skip vote and record flags
  unsigned long long wait_limit_ns;
  int debug_stall;          // test hook: MMA warp withholds its first tile
  unsigned long long* cta_times;  // measurement hook: [cta_cap][3] {start ns, end ns, tiles}, or null
  int cta_cap;
#ifdef LITE_ATTN_TRACE
  long long* trace;         // [4 CTAs][4 roles][8 events][512 tiles] clock64 stamps
#endif
};

// Timing probes for analysis builds (-DLITE_ATTN_TRACE); empty in the library build.
#ifdef LITE_ATTN_TRACE
#define LITE_TRACE(role, ev, t)                                                                        \
  do {                                                                                                 \
    if (p.trace && blockIdx.x < 4 && uint32_t(t) < 512u)                                               \
      p.trace[(((blockIdx.x * 4 + (role)) * 8 + (ev)) * 512) + uint32_t(t)] = clock64();               \
  } while (0)
#else
#define LITE_TRACE(role, ev, t) \
  do {                          \
  } while (0)
#endif

template <int D, int BN>
struct AttnCfg {
  static constexpr int BM = 128;                 // MMA M = TMEM lanes = query rows of a tile slot
  // A kernel query tile has 128 rows. With 64-row Skip-Mask tiles (d = 64) it stacks MR = 2
  // consecutive mask rows (query tiles of the mask): rows 0-63 are mask row 2m, rows 64-127 mask
  // row 2m+1, so every MMA row is a query row. Each half keeps its own Skip-List, running max and
  // QK-Skip vote; a key tile live for only one half computes the other half's rows too and gives
  // them P = 0.
  static constexpr int MR = BM / BN;             // mask rows per kernel query tile: 1 (d=128), 2 (d=64)
  static constexpr int BQ = BM;                  // query rows per kernel query tile (both slots full)
  static constexpr int THREADS = 320;            // producer warp, MMA warp, 2 softmax warpgroups
  static constexpr int NCHUNK = D / 64;          // 128-byte swizzle atoms along d
  static constexpr int Q_CHUNK = BM * 128;       // bytes between d-chunks of a Q tile in smem
  static constexpr int KV_CHUNK = BN * 128;      // bytes between d-chunks of a K or V tile
  static constexpr int Q_BYTES = BM * D * 2;     // one Q tile slot
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr uint32_t Q_TX = BQ * D * 2;   // bytes one Q load delivers
  static constexpr uint32_t KV_TX = BN * D * 2;  // bytes of one K or V tile
  static constexpr int OFF_Q = 0;                // Q_0, Q_1
  static constexpr int OFF_K = OFF_Q + 2 * Q_BYTES;
  static constexpr int OFF_V = OFF_K + 2 * KV_BYTES;
  static constexpr int OFF_CTL = OFF_V + 2 * KV_BYTES;
  static constexpr int CTL_BYTES = 512;
  // O staging for the TMA stores of the epilogue: per softmax warp, 16 rows of D columns, as
  // NCHUNK 128-byte-swizzled panels of 16 x 128 bytes (1024-aligned)
  static constexpr int OST_ROWS = 16;
  static constexpr int OST_PANEL = OST_ROWS * 128;
  static constexpr int OST_WARP = NCHUNK * OST_PANEL;
  static constexpr int OFF_OST = (OFF_CTL + CTL_BYTES + 1023) / 1024 * 1024;
  static constexpr int OST_BYTES = 8 * OST_WARP;
  static constexpr int SMEM_USED = OFF_OST + OST_BYTES + 1024;
  // TMEM columns: S_0 [0, BN), S_1 [BN, 2BN), O_0 [2BN, 2BN+D), O_1 [2BN+D, 2BN+2D)
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t O_COL = 2 * BN;
  static constexpr uint32_t TMEM_COLS = (2 * BN + 2 * D) <= 256 ? 256 : 512;
  // Resident CTAs per SM. A CTA holds TMEM_COLS of the SM's 512 TMEM columns for its whole life.
  // With d = 64 that is 256, so two CTAs run side by side (96 registers a thread, ~83 KB of shared
  // memory each) and hide each other's per-tile latencies. With d = 128 a CTA takes all 512
  // columns, and its shared-memory request is padded so that a second CTA can never be placed
  // on the SM and block in its TMEM allocation.
  static constexpr int CTAS_PER_SM = int(512 / TMEM_COLS);
  static constexpr int SMEM_BYTES =
      CTAS_PER_SM == 2 ? SMEM_USED : (SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024);
  // two CTAs (each also reserving 1 KB of shared memory) within the SM's 228 KB
  static_assert(CTAS_PER_SM == 1 || 2 * (SMEM_BYTES + 1024) <= 228 * 1024, "two CTAs per SM");
  // instruction descriptors, kind::f16: fp32 accumulate (bit 4), bf16 A (bits 7-9) and B (10-12),
  // B major-ness (bit 16), N >> 3 (bits 17-22), M >> 4 (bits 24-28)
  static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                       (uint32_t(BM >> 4) << 24);
  static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                       (uint32_t(D >> 3) << 17) | (uint32_t(BM >> 4) << 24);
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BN == 64 || BN == 128, "tile");
  static_assert(2 * BN + 2 * D <= 512, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  // one TMA box per tile writes its d/64 panels [rows][128 B] back to back
  static_assert(NCHUNK == 1 || (Q_CHUNK == BQ * 128 && KV_CHUNK == BN * 128), "panel strides");
};

// A work item as the producer hands it to the softmax warpgroups: the pair's query tiles, their
// live counts and their first two list entries.
struct PairInfo {
  int row0;      // (b*H + h)*Tq: the head's first mask row; -1 marks the end of the work
  int n[2];      // live key tiles of the pair's two query tiles (0 when the second does not exist)
  int qt[2];     // the two kernel query tiles (qt[1] = Tkq when the item has one)
  int b, h;
  int e[2][2];   // entries 0 and 1 of each query tile's list
  // second mask row of each kernel query tile (MR = 2 only): live count and entries 0 and 1
  int n2[2];
  int e2[2][2];
};

// The query tiles of work item k (0 <= k < ceil(T/2)) of a head under pairing stride s: inside each
// block of 2s tiles, tile r pairs with tile r + s (r < s); the tiles after the last full block pair
// as (t, t+1). Stride 1 pairs 2k with 2k+1. b = -1 when the item has one tile (odd T).
__device__ __forceinline__ void pair_tiles(int k, int T, int s, int& a, int& b) {
  const int full = (T / (2 * s)) * (2 * s);
  if (2 * k < full) {
    const int blk = k / s;
    a = blk * 2 * s + (k - blk * s);
    b = a + s;
  } else {
    a = full + 2 * (k - full / 2);
    b = a + 1;
  }
  if (b >= T) b = -1;
}

// Per union tile, what the producer tells the MMA thread (one 32-bit word in a 4-slot ring).
constexpr uint32_t kLive0 = 1u, kLive1 = 2u;        // live for query tile 0 / 1
constexpr uint32_t kFirst0 = 4u, kFirst1 = 8u;      // first live tile of query tile 0 / 1 in the item
constexpr uint32_t kLast0 = 16u, kLast1 = 32u;      // last live tile of query tile 0 / 1 in the item
constexpr uint32_t kItemFirst = 64u;                // first union tile of an item
constexpr uint32_t kItemLast = 128u;                // last union tile of an item
constexpr uint32_t kEnd = 256u;                     // no more tiles (the bundle carries the last V)
constexpr int kItemShift = 12;                      // bits 12..31: the item's number in this CTA

// Control block in shared memory (barriers are 8-byte mbarrier objects).
struct alignas(8) AttnCtl {
  uint64_t q_full, q_empty;          // the pair's Q tiles landed / read by the item's last QK
  uint64_t kv_full[2];               // bundle u landed: K_u (stage u%2) and V_{u-1} (stage (u-1)%2)
  uint64_t kv_free[2];               // the QKs of union tile u (and every MMA before them) finished
  uint64_t s_full[2];                // S_g ready (one phase per live tile of query tile g)
  uint64_t p_full[2];                // P_g written (one phase per live tile of query tile g)
  uint64_t pv_done[2];               // last PV_g of an item finished (accumulator g)
  uint64_t o_free[2];                // group g's epilogue has read O_g (one phase per item)
  uint64_t item_full[2], item_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  uint32_t tiles;                    // live (query tile, key tile) pairs processed (measurement hook)
  uint32_t ring[4];                  // per union tile u (slot u%4): the flags above
  PairInfo info[2];                  // handed-out items
};
// UMMA shared-memory descriptor, 128-byte swizzle (layout type 2, bits 61-63), version 1 (bit 46).
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// 2^x on the FMA/ALU pipes, for the share of the exponentials taken off the MUFU unit.
// Range reduction in the manner of Cody and Waite: adding 1.5*2^23 rounds x to the nearest integer
// n in the low mantissa bits of t, f = x - n lies in [-1/2, 1/2], 2^f comes from a cubic, and n is
// added to the exponent field. The cubic interpolates 2^f at the four Chebyshev nodes of
// [-1/2, 1/2] (max relative error 1.0e-4, far below the 2^-9 rounding of the bf16 P it feeds).
// x is clamped at -126 so the exponent field stays valid; results below 2^-126 are immaterial here.
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -126.0f);
  const float t = x + 12582912.0f;
  const float f = x - (t - 12582912.0f);
  const float p = fmaf(fmaf(fmaf(0.05583828315138817f, f, 0.2426394820213318f), f, 0.6931367516517639f), f,
                       0.9999245405197144f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// The same 2^x for two values with packed fp32x2 arithmetic (identical float32 steps, so identical
// results): 12 instructions for two exponentials instead of two MUFU operations.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
  const float2 n = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
  const float2 f = __ffma2_rn(n, make_float2(-1.0f, -1.0f), x);
  float2 q = __ffma2_rn(make_float2(0.05583828315138817f, 0.05583828315138817f), f,
                        make_float2(0.2426394820213318f, 0.2426394820213318f));
  q = __ffma2_rn(q, f, make_float2(0.6931367516517639f, 0.6931367516517639f));
  q = __ffma2_rn(q, f, make_float2(0.9999245405197144f, 0.9999245405197144f));
  return make_float2(__int_as_float(__float_as_int(q.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(q.y) + (__float_as_int(t.y) << 23)));
}

struct Waiter {
  volatile int* abort;
  int* status;
  unsigned long long limit;

  // Wait for completion of the phase with `parity`; false on timeout or when another role gave up.
  __device__ __forceinline__ bool wait(uint32_t bar, uint32_t parity) const {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    const uint64_t t0 = ptx::globaltimer();
    while (true) {
      if (ptx::mbar_try_wait(bar, parity)) return true;
      if (*abort) return false;
      if (ptx::globaltimer() - t0 > limit) {
        give_up();
        return false;
      }
    }
  }
  // Same, ignoring the abort flag (used only to drain in-flight copies before exit).
  __device__ __forceinline__ bool wait_drain(uint32_t bar, uint32_t parity) const {
    const uint64_t t0 = ptx::globaltimer();
    while (!ptx::mbar_try_wait(bar, parity)) {
      if (ptx::globaltimer() - t0 > limit) {
        give_up();
        return false;
      }
    }
    return true;
  }
  __device__ __forceinline__ void give_up() const { stop(kStatusTimeout); }
  __device__ __forceinline__ void fail_check() const { stop(kStatusCheck); }
  __device__ __forceinline__ void stop(int code) const {
    *abort = 1;
    atomicCAS(status, 0, code);
    __threadfence_block();
  }
};

// idx-th live key tile of a row, with its kListNoFlag tag (dense: Tk-1, Tk-2, ..., untagged)
__device__ __forceinline__ int key_entry(const AttnParams& p, int row, int idx) {
  return p.list ? int(p.list[size_t(row) * p.Tk + idx]) : (p.Tk - 1 - idx);
}

// Work item `item` (in hand-out order) decoded: the pair's rows, live counts and first entries.
// Returns false (and a pair with no live tiles) when the work order or a live count is out of range.
template <int MR>
__device__ __forceinline__ bool decode_pair(const AttnParams& p, int item, int stride, PairInfo& it) {
  const int pair = p.order ? p.order[item] : item;
  if (pair < 0 || pair >= p.n_items) {
    it.row0 = 0;
    it.n[0] = it.n[1] = 0;
    it.n2[0] = it.n2[1] = 0;
    return false;
  }
  const int bh = pair / p.Pq;
  const int k = pair - bh * p.Pq;
  it.b = bh / p.H;
  it.h = bh - it.b * p.H;
  it.row0 = bh * p.Tq;
  int a, b;
  pair_tiles(k, p.Tkq, stride, a, b);
  it.qt[0] = a;
  it.qt[1] = b >= 0 ? b : p.Tkq;
  bool ok = true;
  int n[2][MR];
#pragma unroll
  for (int g = 0; g < 2; ++g)
#pragma unroll
    for (int hf = 0; hf < MR; ++hf) {
      const int mrow = it.qt[g] * MR + hf;
      const bool exists = it.qt[g] < p.Tkq && mrow < p.Tq;
      int c = !exists ? 0 : (p.counts ? p.counts[it.row0 + mrow] : p.Tk);
      if (c < 0 || c > p.Tk) {
        ok = false;
        c = 0;
      }
      n[g][hf] = c;
    }
#pragma unroll
  for (int g = 0; g < 2; ++g)
#pragma unroll
    for (int hf = 0; hf < MR; ++hf) {
      const int c = ok ? n[g][hf] : 0;
      const int r = it.row0 + it.qt[g] * MR + hf;
      const int e0 = c > 0 ? key_entry(p, r, 0) : 0;
      const int e1 = c > 1 ? key_entry(p, r, 1) : 0;
      if (hf == 0) {
        it.n[g] = c;
        it.e[g][0] = e0;
        it.e[g][1] = e1;
      } else {
        it.n2[g] = c;
        it.e2[g][0] = e0;
        it.e2[g][1] = e1;
      }
    }
  if constexpr (MR == 1) it.n2[0] = it.n2[1] = 0;
  return ok;
}

// Walks one query tile's descending list; the entry after the current one is kept prefetched.
struct ListCursor {
  int row, n, i;
  int cur, nxt;  // raw entries i and i+1
  int above;     // key tile of the previously consumed entry (Tk before the first)
  __device__ __forceinline__ int head() const { return i < n ? (cur & kListIndexMask) : -1; }
  // The current entry is well formed: only the index and no-flag bits set, index below both Tk and
  // the previous entry's (lists are strictly descending).
  __device__ __forceinline__ bool head_ok() const {
    return (cur & ~(kListIndexMask | kListNoFlag)) == 0 && (cur & kListIndexMask) < above;
  }
  __device__ __forceinline__ void advance(const AttnParams& p) {
    above = cur & kListIndexMask;
    ++i;
    cur = nxt;
    if (i + 1 < n) nxt = key_entry(p, row, i + 1);
  }
};

// Lazy rescale: the exponent reference of a row moves only when a tile's max exceeds it by more
// than this many log2 units, so P stays below 2^kRescaleLog2. Measured on this B200: a larger
// threshold rescales O less often, but P values far above 1 in a single long accumulation raise
// the output error (8 gives ~15% more RMS error than 0); 2 keeps the error at the level of an
// exact running max within ~1% of the speed of 8.
constexpr float kRescaleLog2 = 2.0f;

// Item parity and "not the CTA's first item" travel in the ring word next to the tile flags.
constexpr uint32_t kItemOdd = 512u, kItemAfterFirst = 1024u;

template <int D, int BN>
__global__ void __launch_bounds__(320, AttnCfg<D, BN>::CTAS_PER_SM)
    lite_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const AttnParams p) {
  using C = AttnCfg<D, BN>;
  static_assert(sizeof(AttnCtl) <= C::CTL_BYTES, "control block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnCtl* ctl = reinterpret_cast<AttnCtl*>(smem + C::OFF_CTL);
  const uint32_t sQ = ptx::smem_addr(smem + C::OFF_Q);
  const uint32_t sK = ptx::smem_addr(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_addr(smem + C::OFF_V);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

#define BAR(x) ptx::smem_addr(&ctl->x)

  const uint64_t t_start = ptx::globaltimer();
  if (threadIdx.x == 0) {
    ptx::mbar_init(BAR(q_full), 1);
    ptx::mbar_init(BAR(q_empty), 1);
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(BAR(kv_full[b]), 1);
      ptx::mbar_init(BAR(kv_free[b]), 1);
      ptx::mbar_init(BAR(s_full[b]), 1);
      ptx::mbar_init(BAR(p_full[b]), 128);
      ptx::mbar_init(BAR(pv_done[b]), 1);
      ptx::mbar_init(BAR(o_free[b]), 128);
      ptx::mbar_init(BAR(item_full[b]), 1);
      ptx::mbar_init(BAR(item_empty[b]), 8);  // one lane of each softmax warp
    }
    ptx::mbar_init(BAR(drain), 1);
    ctl->abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    ptx::prefetch_tmap(&tmO);
  }
  if (warp == 1) {
    ptx::tmem_alloc(ptx::smem_addr(&ctl->tmem_base), C::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const Waiter wt{&ctl->abort, p.status, p.wait_limit_ns};

  // Barrier phases. Union tiles u are numbered over all items this CTA processes; bundle u uses
  // kv_full / kv_free slot u%2 and ring slot u%4. s_full[g] and p_full[g] complete once per live
  // tile of query tile g, q_full / q_empty and o_free[g] once per item with tiles, pv_done[g] once
  // per item in which query tile g has a live tile. Every waiter either observes each phase of a
  // barrier in order, or the order of the MMA thread's commits keeps the barrier within one phase
  // of the awaited one (the argument is written at each wait), so the parity waits are exact.
  if (warp == 0) {
    // ------------------------------------------------------------------------- TMA producer
    // Bundle u carries K_u (stage u%2) and V_{u-1} (stage (u-1)%2). K stage u%2 was last read by
    // the QKs of union tile u-2; V stage (u-1)%2 by the PVs of union tile u-3, which the MMA thread
    // issues before those QKs. So one wait (kv_free of u-2) frees both, and the MMA thread waits
    // once per union tile. A last bundle carries only the final V, with the end mark.
    if (lane == 0) {
      uint32_t u = 0, items = 0, qn = 0, live_pairs = 0;
      bool ok = true;
      const int stride = p.pair_stride_ptr ? *p.pair_stride_ptr : p.pair_stride;
      // last armed phase of each full barrier, so that every issued load can be drained at exit
      bool q_armed = false, kv_armed[2] = {false, false};
      uint32_t q_par = 0, kv_par[2] = {0, 0};
      int pj = 0, ph = 0, pb = 0;  // coordinates of union tile u-1
      bool v_needed = false;       // union tile u-1 had a live tile, so bundle u carries V_{u-1}
      // kv_free of slot u%2 next completes with the QKs of union tile u, which need this bundle
      auto bundle = [&](bool with_k, int j, int h, int b, uint32_t flags) -> bool {
        LITE_TRACE(0, 0, u);
        if (u >= 2 && !wt.wait(BAR(kv_free[u & 1]), ((u - 2) >> 1) & 1)) return false;
        // the ring word is written before the bundle's barrier is armed (release), and read by the
        // MMA thread after it waited on that barrier (acquire)
        ctl->ring[u & 3] = flags;
        const uint32_t bar = BAR(kv_full[u & 1]);
        ptx::mbar_arrive_expect_tx(bar, (with_k ? C::KV_TX : 0u) + (v_needed ? C::KV_TX : 0u));
        if (with_k) ptx::tma_load_5d(sK + (u & 1) * C::KV_BYTES, &tmK, bar, 0, j * BN, 0, h, b);
        if (v_needed) ptx::tma_load_5d(sV + ((u - 1) & 1) * C::KV_BYTES, &tmV, bar, 0, pj * BN, 0, ph, pb);
        v_needed = with_k;  // every union tile with a K load has a live tile
        kv_armed[u & 1] = true;
        kv_par[u & 1] = (u >> 1) & 1;
        LITE_TRACE(0, 1, u);
        pj = j;
        ph = h;
        pb = b;
        ++u;
        return true;
      };
      while (ok) {
        const int slot = items & 1;
        if (items >= 2) ok = wt.wait(BAR(item_empty[slot]), ((items >> 1) - 1) & 1);
        if (!ok) break;
        // dynamic hand-out in schedule order; without a counter, static striding (uniform items)
        int item = p.work_counter ? atomicAdd(p.work_counter, 1) : int(blockIdx.x + items * gridDim.x);
        if (item >= p.n_items) item = -1;
        PairInfo it{};
        it.row0 = -1;
        bool good = true;
        if (item >= 0) good = stride >= 1 && decode_pair<C::MR>(p, item, stride, it);
        if (!good) it.row0 = -1;  // the softmax groups stop as at the end of the work
        ctl->info[slot] = it;
        ptx::mbar_arrive(BAR(item_full[slot]));
        ++items;
        if (!good) {
          wt.fail_check();  // work order or live count out of range
          ok = false;
          break;
        }
        if (item < 0) break;
        const int gn[2] = {it.n[0] + it.n2[0], it.n[1] + it.n2[1]};  // live tiles per kernel query tile
        if (gn[0] + gn[1] == 0) {
          // An item without tiles needs no bundle. But a softmax group may still wait, in the
          // epilogue of its previous item, for the PV of that item's last union tile, which the MMA
          // thread issues with the next bundle; and before this producer hands out two more items,
          // both groups must have read this one. So the pending PVs are flushed now, by a bundle
          // with V only and no live tile.
          if (v_needed) ok = bundle(false, 0, 0, 0, 0u);
          continue;
        }
        // the pair's Q tiles; q_empty is committed after the item's last QK
        if (qn >= 1) ok = wt.wait(BAR(q_empty), (qn - 1) & 1);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(BAR(q_full), (gn[0] > 0 ? C::Q_TX : 0u) + (gn[1] > 0 ? C::Q_TX : 0u));
        for (int g = 0; g < 2; ++g)
          if (gn[g] > 0)
            ptx::tma_load_5d(sQ + g * C::Q_BYTES, &tmQ, BAR(q_full), 0, it.qt[g] * C::BQ, 0, it.h, it.b);
        q_armed = true;
        q_par = qn & 1;
        const uint32_t item_bits = ((qn & 1) ? kItemOdd : 0u) | (qn >= 1 ? kItemAfterFirst : 0u);
        uint32_t f = kItemFirst;
        if constexpr (C::MR == 1) {
        // the union of the two descending lists, highest key tile first
        ListCursor c0{it.row0 + it.qt[0], it.n[0], 0, it.e[0][0], it.e[0][1], p.Tk};
        ListCursor c1{it.row0 + it.qt[1], it.n[1], 0, it.e[1][0], it.e[1][1], p.Tk};
        while (ok) {
          const int h0 = c0.head(), h1 = c1.head();
          const int j = max(h0, h1);
          if ((h0 == j && !c0.head_ok()) || (h1 == j && !c1.head_ok())) {
            wt.fail_check();  // malformed or not strictly descending
            ok = false;
            break;
          }
          f |= item_bits;
          if (h0 == j) f |= kLive0 | (c0.i == 0 ? kFirst0 : 0u) | (c0.i == c0.n - 1 ? kLast0 : 0u);
          if (h1 == j) f |= kLive1 | (c1.i == 0 ? kFirst1 : 0u) | (c1.i == c1.n - 1 ? kLast1 : 0u);
          if (h0 == j) c0.advance(p);
          if (h1 == j) c1.advance(p);
          const bool last = c0.head() < 0 && c1.head() < 0;
          if (last) f |= kItemLast;
          ok = bundle(true, j, it.h, it.b, f);
          if (last) break;
          f = 0u;
        }
        } else {
        // Stacked rows: kernel query tile g has two mask rows, each with its own list. The key tiles
        // of the item are the union of the four lists; tile j is computed for kernel tile g when it
        // is live for either of g's rows.
        ListCursor cur[2][2] = {
            {{it.row0 + it.qt[0] * 2, it.n[0], 0, it.e[0][0], it.e[0][1], p.Tk},
             {it.row0 + it.qt[0] * 2 + 1, it.n2[0], 0, it.e2[0][0], it.e2[0][1], p.Tk}},
            {{it.row0 + it.qt[1] * 2, it.n[1], 0, it.e[1][0], it.e[1][1], p.Tk},
             {it.row0 + it.qt[1] * 2 + 1, it.n2[1], 0, it.e2[1][0], it.e2[1][1], p.Tk}}};
        bool started[2] = {false, false};
        while (ok) {
          int j = -1;
#pragma unroll
          for (int g = 0; g < 2; ++g) j = max(j, max(cur[g][0].head(), cur[g][1].head()));
          f |= item_bits;
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            bool live = false;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
              if (cur[g][hf].head() == j) {
                if (!cur[g][hf].head_ok()) ok = false;  // malformed or not strictly descending
                cur[g][hf].advance(p);
                live = true;
              }
            if (live) {
              f |= (kLive0 << g) | (started[g] ? 0u : (kFirst0 << g));
              started[g] = true;
              if (cur[g][0].head() < 0 && cur[g][1].head() < 0) f |= kLast0 << g;
            }
          }
          if (!ok) {
            wt.fail_check();
            break;
          }
          const bool last = cur[0][0].head() < 0 && cur[0][1].head() < 0 && cur[1][0].head() < 0 &&
                            cur[1][1].head() < 0;
          if (last) f |= kItemLast;
          ok = bundle(true, j, it.h, it.b, f);
          if (last) break;
          f = 0u;
        }
        }
        live_pairs += uint32_t(it.n[0] + it.n[1] + it.n2[0] + it.n2[1]);
        ++qn;
      }
      ctl->tiles = live_pairs;
      if (ok) bundle(false, 0, 0, 0, kEnd);  // the last union tile's V, and the end mark
      // Drain: every issued TMA load has landed before this thread leaves (no other thread arms these
      // barriers, so the last armed phase is the one to wait for).
      if (q_armed) wt.wait_drain(BAR(q_full), q_par);
      for (int b = 0; b < 2; ++b)
        if (kv_armed[b]) wt.wait_drain(BAR(kv_full[b]), kv_par[b]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------------- MMA issuer
    // Per union tile u, once bundle u landed: for g = 0, 1, PV_g(u-1) if u-1 was live for query
    // tile g, then QK_g(u) if u is live for it. QK_g(u) reuses S buffer g after PV_g(u-1) read the
    // P in it, and the next QK_g needs the softmax's P_g of this tile first: MMAs of this thread
    // run in issue order. One commit per union tile frees the bundle's stages.
    if (lane == 0) {
      uint32_t u = 0;
      uint32_t pc[2] = {0, 0};  // P phases consumed per query tile
      uint32_t prev = 0;        // flags of union tile u-1
      bool ok = true;
      // 128B-swizzled K-major operands advance 32 bytes (>> 4 = 2) per K=16 step inside an atom;
      // V (MN-major) advances 16 rows = 2048 bytes (>> 4 = 128) per step.
      const uint64_t q_desc0 = umma_desc_sw128(sQ, 16, 1024);
      const uint64_t k_desc0 = umma_desc_sw128(sK, 16, 1024);
      const uint64_t v_desc0 = umma_desc_sw128(sV, C::KV_CHUNK, 1024);
      const uint32_t bar_kv = BAR(kv_full[0]), bar_free = BAR(kv_free[0]);
      if (p.debug_stall) {
        // test hook: withhold all work until the other roles give up
        const uint64_t s0 = ptx::globaltimer();
        while (!ctl->abort && ptx::globaltimer() - s0 < 4ull * p.wait_limit_ns) {
        }
        if (!ctl->abort) wt.give_up();
        ok = false;
      }
      while (ok) {
        // kv_full of slot u%2 next completes for bundle u+2, loaded after the QKs of u finished
        LITE_TRACE(1, 0, u);
        if (!wt.wait(bar_kv + (u & 1) * 8, (u >> 1) & 1)) break;
        LITE_TRACE(1, 1, u);
        const uint32_t f = ctl->ring[u & 3];
        ptx::tc_fence_after();
        // q_full completes once per item; the next load waits for this item's q_empty commit
        bool need_q = (f & kItemFirst) != 0u;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          if (prev & (kLive0 << g)) {
            // The first PV of query tile g in an item overwrites O_g: the previous item's epilogue
            // of group g must have read it (o_free[g]: one phase per item, exact because the next
            // phase needs this item's PVs). p_full[g] next completes for g's next live tile, whose
            // S needs a QK issued after this PV.
            if ((prev & (kFirst0 << g)) && (prev & kItemAfterFirst) &&
                !wt.wait(BAR(o_free[g]), (prev & kItemOdd) ? 0u : 1u)) {
              ok = false;
              break;
            }
            if (!wt.wait(BAR(p_full[g]), pc[g] & 1)) {
              ok = false;
              break;
            }
            ++pc[g];
            ptx::tc_fence_after();
            const uint32_t p_tmem = tmem + C::S_COL + g * BN;
            const uint32_t o_tmem = tmem + C::O_COL + g * D;
            const uint64_t vd = v_desc0 + uint64_t((((u - 1) & 1) * C::KV_BYTES) >> 4);
            const bool fresh = (prev & (kFirst0 << g)) != 0u;
#pragma unroll
            for (int kk = 0; kk < BN / 16; ++kk)
              ptx::mma_ts(o_tmem, p_tmem + kk * 8, vd + uint64_t(kk * 128), C::IDESC_PV, (fresh && kk == 0) ? 0u : 1u);
            // the epilogue of group g waits for the item's last PV into its accumulator
            if (prev & (kLast0 << g)) ptx::mma_commit(BAR(pv_done[g]));
          }
          if (f & (kLive0 << g)) {
            if (need_q) {
              if (!wt.wait(BAR(q_full), (f & kItemOdd) ? 1u : 0u)) {
                ok = false;
                break;
              }
              ptx::tc_fence_after();
              need_q = false;
            }
            const uint64_t qd = q_desc0 + uint64_t((g * C::Q_BYTES) >> 4);
            const uint64_t kd = k_desc0 + uint64_t(((u & 1) * C::KV_BYTES) >> 4);
            const uint32_t s_tmem = tmem + C::S_COL + g * BN;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = uint64_t((kk >> 2) * (C::Q_CHUNK >> 4) + (kk & 3) * 2);
              const uint64_t offk = uint64_t((kk >> 2) * (C::KV_CHUNK >> 4) + (kk & 3) * 2);
              ptx::mma_ss(s_tmem, qd + off, kd + offk, C::IDESC_QK, kk > 0 ? 1u : 0u);
            }
            ptx::mma_commit(BAR(s_full[g]));
          }
        }
        LITE_TRACE(1, 2, u);
        if (!ok || (f & kEnd)) break;
        ptx::mma_commit(bar_free + (u & 1) * 8);
        if (f & kItemLast) ptx::mma_commit(BAR(q_empty));
        prev = f;
        ++u;
      }
      // all issued tensor-core work must finish before TMEM is released
      ptx::mma_commit(BAR(drain));
      wt.wait_drain(BAR(drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------- softmax warpgroups
    const int grp = (warp - 2) >> 2;                // query tile qt[grp] of each pair
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;              // TMEM lane = row inside the tile slot
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const uint32_t gbar = 1 + grp;                  // named barrier of this warpgroup (128 threads)
    uint8_t* stage = smem + C::OFF_OST + (grp * 4 + quarter) * C::OST_WARP;
    const int wrow = quarter * 32;                  // first tile row of this warp's lanes
    uint32_t tg = 0, items = 0, pv_phase = 0;
    while (true) {
      const int slot = items & 1;
      bool ok = wt.wait(BAR(item_full[slot]), (items >> 1) & 1);
      const PairInfo it = ctl->info[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(BAR(item_empty[slot]));
      ++items;
      if (!ptx::named_bar_and(gbar, 128, ok) || it.row0 < 0) break;
      const int qi = it.qt[grp];  // Tkq when the item has no second query tile
      const int n = it.n[grp] + it.n2[grp];  // live tiles of the kernel query tile's mask rows
      const int half = C::MR == 1 ? 0 : (r >> 6);  // stacked rows: which mask row this thread's row is in
      const int row = it.row0 + qi * C::MR;         // first mask row of the kernel query tile
      const int vrow = row + half;                  // this thread's mask row
      const int rq = r;  // row inside the kernel query tile
      const int n_row = qi * C::BQ + rq;
      const bool valid_row = qi < p.Tkq && rq >= 0 && rq < C::BQ && n_row < p.Nq;
      const size_t o_off = (size_t(it.b) * p.Nq + n_row) * p.H + it.h;
      const bool any = it.n[0] + it.n[1] + it.n2[0] + it.n2[1] > 0;
      if (n == 0) {
        // a query tile without live key tiles: O = 0, lse = -inf; o_free keeps one phase per item
        if (valid_row) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + o_off * D);
          for (int x = 0; x < D / 8; ++x) dst[x] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[(size_t(it.b) * p.H + it.h) * p.Nq + n_row] = -INFINITY;
        }
        if (any) ptx::mbar_arrive(BAR(o_free[grp]));
        continue;
      }
      float m_true = -INFINITY;  // running max over the tile's earlier live key tiles (log2 units)
      float m_used = -INFINITY;  // exponent reference (lazy rescale)
      float l = 0.f;             // row sum relative to m_used
      // One live key tile j of the kernel query tile (t counts the group's tiles over all items,
      // idx within this item); live_me is false only for a stacked row whose mask row skips j.
      auto tile = [&](uint32_t t, int j, bool may_flag, bool live_me, int idx) {
          if (r == 0) LITE_TRACE(2 + grp, 0, t);
          // s_full[g] next completes for g's next live tile, whose QK follows this tile's PV
          wt.wait(BAR(s_full[grp]), t & 1);
          __syncwarp();
          ptx::tc_fence_after();
          float loc = -INFINITY;  // the tile's row max (log2 units)
          if (!live_me) {
            // (stacked rows only) key tile j is skipped for this row's mask row: P = 0 for the row
            const uint32_t s_tmem = tmem + lane_base + C::S_COL + grp * BN;
            uint32_t zero[16];
  #pragma unroll
            for (int x = 0; x < 16; ++x) zero[x] = 0u;
  #pragma unroll
            for (int c = 0; c < BN / 32; ++c) ptx::tmem_st16(s_tmem + c * 16, zero);
            ptx::tmem_wait_st();
          }
          if (live_me) {
          const uint32_t s_tmem = tmem + lane_base + C::S_COL + grp * BN;
          // the whole S row is read once and stays in registers for the max and the exponentials
          uint32_t sr[BN];
  #pragma unroll
          for (int c = 0; c < BN / 32; ++c)
            ptx::tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
          ptx::tmem_wait_ld();
          if (r == 0) LITE_TRACE(2 + grp, 1, t);
          float s[BN];
  #pragma unroll
          for (int x = 0; x < BN; ++x) s[x] = __uint_as_float(sr[x]);
          const int valid_cols = min(BN, p.Nk - j * BN);
          if (valid_cols < BN) {
            // key columns past Nk (zero-filled by TMA) take no part in max, sum or PV
  #pragma unroll
            for (int x = 0; x < BN; ++x)
              if (x >= valid_cols) s[x] = -INFINITY;
          }
          float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
  #pragma unroll
          for (int x = 0; x < BN; x += 8) {
            m0 = ptx::fmax3(m0, s[x], s[x + 1]);
            m1 = ptx::fmax3(m1, s[x + 2], s[x + 3]);
            m2 = ptx::fmax3(m2, s[x + 4], s[x + 5]);
            m3 = ptx::fmax3(m3, s[x + 6], s[x + 7]);
          }
          loc = ptx::fmax3(m0, m1, fmaxf(m2, m3)) * p.scale_log2;
          // lazy rescale of the accumulator: move the reference only when the tile max exceeds it by
          // more than kRescaleLog2. O itself is rescaled after the exponentials below, when the S row
          // no longer occupies registers (doing it here made the compiler spill S on every tile).
          const bool need = loc > m_used + kRescaleLog2;
          float alpha = 1.f;
          if (need) {
            alpha = ptx::ex2(m_used - loc);
            m_used = loc;
            l *= alpha;
          }
          // P = 2^(s*scale*log2e - m_used) as bf16 pairs over the S columns (chunk c of 32 key
          // columns -> TMEM columns [16c, 16c+16)), released to the MMA thread in one piece. Packed
          // fp32x2 arithmetic for the affine step and the row sum; one column pair in sixteen is
          // exponentiated on the FMA pipe, the rest on MUFU (measured: 1/16 and none beat 1/8 and 1/4
          // by ~1% once the O rescale left the S -> P path).
          const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
          const float2 nm2 = make_float2(-m_used, -m_used);
          float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  #pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            uint32_t pk[16];
  #pragma unroll
            for (int x = 0; x < 16; ++x) {
              const float2 a = __ffma2_rn(make_float2(s[32 * c + 2 * x], s[32 * c + 2 * x + 1]), sc2, nm2);
              const float2 pp = (x == 15) ? exp2_poly2(a) : make_float2(ptx::ex2(a.x), ptx::ex2(a.y));
              acc[x & 3] = __fadd2_rn(acc[x & 3], pp);
              __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
              pk[x] = *reinterpret_cast<uint32_t*>(&h2);
            }
            ptx::tmem_st16(s_tmem + c * 16, pk);
          }
          // The previous PV into O_g was issued before this tile's QK, so it has completed now that S
          // is ready; the rescaled O is stored before P is released (both stores are waited for below).
          if (__any_sync(0xffffffffu, need) && idx >= 1) {
            const uint32_t o_tmem = tmem + lane_base + C::O_COL + grp * D;
  #pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
              uint32_t rr[32];
              ptx::tmem_ld32(o_tmem + c * 32, rr);
              ptx::tmem_wait_ld();
  #pragma unroll
              for (int x = 0; x < 32; ++x) rr[x] = __float_as_uint(__uint_as_float(rr[x]) * alpha);
              ptx::tmem_st32(o_tmem + c * 32, rr);
            }
          }
          ptx::tmem_wait_st();
          const float2 acc2 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
          l += acc2.x + acc2.y;
          }
          ptx::tc_fence_before();
          ptx::mbar_arrive(BAR(p_full[grp]));
          if (r == 0) LITE_TRACE(2 + grp, 2, t);
          if (p.skip_test && live_me) {
            // QK-Skip, off the path from S to P: flag key tile j when loc - m < tau for every valid
            // row of the mask row, m the running max over the row's earlier live key tiles. With
            // stacked rows each 64-row half votes on its own named barrier (its two warps).
            const bool pred = !valid_row || (loc - m_true < p.tau_log2);
            const bool flag = C::MR == 1 ? ptx::named_bar_and(gbar, 128, pred)
                                         : ptx::named_bar_and(3 + 2 * grp + half, 64, pred);
            if (flag && may_flag && (r & (C::BM / C::MR - 1)) == 0 && p.mask_out && !ctl->abort)
              atomicOr(p.mask_out + size_t(vrow) * p.W + (j >> 5), 1u << (j & 31));
          }
          if (r == 0) LITE_TRACE(2 + grp, 3, t);
          m_true = fmaxf(m_true, loc);
      };
      if constexpr (C::MR == 1) {
        int e_cur = it.e[grp][0], e_nxt = it.e[grp][1];
        for (int idx = 0; idx < n; ++idx) {
          const int j = e_cur & kListIndexMask;
          const bool may_flag = !(e_cur & kListNoFlag);
          e_cur = e_nxt;
          if (idx + 2 < n) e_nxt = key_entry(p, row, idx + 2);  // prefetch
          tile(tg + idx, j, may_flag, true, idx);
        }
        tg += n;
      } else {
        // the union of the kernel query tile's two mask rows' lists, highest key tile first
        const int mi = half, oi = 1 - half;
        const int nm = mi == 0 ? it.n[grp] : it.n2[grp], no = oi == 0 ? it.n[grp] : it.n2[grp];
        ListCursor mine{row + mi, nm, 0, mi == 0 ? it.e[grp][0] : it.e2[grp][0], mi == 0 ? it.e[grp][1] : it.e2[grp][1],
                        p.Tk};
        ListCursor other{row + oi, no, 0, oi == 0 ? it.e[grp][0] : it.e2[grp][0], oi == 0 ? it.e[grp][1] : it.e2[grp][1],
                         p.Tk};
        int idx = 0;
        while (true) {
          const int hm = mine.head(), ho = other.head();
          if (hm < 0 && ho < 0) break;
          const int j = max(hm, ho);
          const bool live_me = hm == j;
          const bool may_flag = live_me && !(mine.cur & kListNoFlag);
          if (live_me) mine.advance(p);
          if (ho == j) other.advance(p);
          tile(tg + idx, j, may_flag, live_me, idx);
          ++idx;
        }
        tg += idx;
      }
      // Epilogue: wait for the item's last PV into O_g, normalise, and write the rows (bf16) out
      // through shared memory: each warp stages the rows of lanes 0-15, then those of lanes 16-31,
      // and its lane 0 issues one TMA store per half (rows past Nq are clipped by the TMA unit). A
      // staging half is rewritten only after its previous store has read it. pv_done[g] completes
      // once per item in which query tile g has a live tile.
      wt.wait(BAR(pv_done[grp]), pv_phase & 1);
      ++pv_phase;
      ptx::tc_fence_after();
      // a stacked row whose mask row has no live tile in the item: O = 0, lse = -inf
      const float inv_l = (C::MR == 1 || l > 0.f) ? 1.f / l : 0.f;
      uint32_t ow[D / 2];  // the row's D columns, packed in bf16 pairs
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        ptx::tmem_ld32(tmem + lane_base + C::O_COL + grp * D + c * 32, rr);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(rr[2 * x]) * inv_l,
                                                    __uint_as_float(rr[2 * x + 1]) * inv_l);
          ow[c * 16 + x] = *reinterpret_cast<uint32_t*>(&h2);
        }
      }
      ptx::tc_fence_before();
      ptx::mbar_arrive(BAR(o_free[grp]));
      const int srow = lane & (C::OST_ROWS - 1);
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        if (lane == 0) ptx::bulk_wait_group_read0();
        __syncwarp();
        if ((lane >> 4) == part) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c) {
            // 16-byte chunk c of the row: panel c/8, 128-byte swizzle (chunk ^ row % 8) inside it
            const int x = c & 7;
            *reinterpret_cast<uint4*>(stage + (c >> 3) * C::OST_PANEL + srow * 128 + ((x ^ (srow & 7)) << 4)) =
                make_uint4(ow[4 * c], ow[4 * c + 1], ow[4 * c + 2], ow[4 * c + 3]);
          }
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        const int row_in_tile = wrow + part * C::OST_ROWS;
        if (lane == 0 && qi < p.Tkq && row_in_tile < C::BQ && qi * C::BQ + row_in_tile < p.Nq) {
          ptx::tma_store_5d(&tmO, ptx::smem_addr(stage), 0, qi * C::BQ + row_in_tile, 0, it.h, it.b);
          ptx::bulk_commit_group();
        }
      }
      if (valid_row && p.lse)
        p.lse[(size_t(it.b) * p.H + it.h) * p.Nq + n_row] =
            (C::MR == 1 || l > 0.f) ? (m_used + __log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
    // the staged O rows must have been written out before the CTA (and its shared memory) ends
    if (lane == 0) ptx::bulk_wait_group0();
    __syncwarp();
  }
#undef BAR

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0 && p.cta_times && int(blockIdx.x) < p.cta_cap) {
    unsigned long long* rec = p.cta_times + 3 * size_t(blockIdx.x);
    rec[0] = t_start;
    rec[1] = ptx::globaltimer();
    rec[2] = ctl->tiles;
  }
}

}  // namespace lite
