// attn_kernel.cuh -- persistent block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA per SM walks a list of work items; an item is one query tile of one (b, h). For an item
// it streams only the live key tiles of that query tile (LiteAttention README, "Full-Stage
// Elimination": a skipped tile costs no K/V load, no QK^T, no softmax, no PV), from the highest
// key-tile index down (README, must_do_list: "we iterate in reverse order inside of the kernel").
// Queries and keys may differ in length (README, LSE section: partial attentions such as text-to-
// video over a subset of the keys); a key tile that a must-do range keeps live carries a tag in its
// list entry and is computed but never flagged.
//
// Warp roles (320 threads):
//   warp 0       TMA producer: Q once per item; per live tile K_j into a 2-stage ring and V_j into
//                a 3-stage ring (separate barriers, so S = QK^T never waits for V).
//   warp 1       TMEM allocator and single-thread tcgen05 MMA issuer, in the order
//                QK_0, QK_1, PV_0, QK_2, PV_1, ... over the live tiles of consecutive items:
//                  S_t = Q K_t^T  (SS form) into TMEM buffer t%2,
//                  O_{t%2} += P_t V_t (TS form: P read from TMEM, V from shared memory).
//   warps 2..5   softmax warpgroup 0: the tiles t with t%2 == 0;  warps 6..9: warpgroup 1, t%2 == 1.
//                One thread per query row (TMEM lane). The two groups work on consecutive tiles at
//                the same time, each with its own running exponent reference, row sum and O
//                accumulator; the epilogue combines the two partial softmaxes exactly. Per tile:
//                row max; the QK-Skip vote (skill page "Lite Attention Temporal Sparse", Core
//                Concept: a tile whose local max score is far below the cumulative max is
//                flagged) against the running max over ALL earlier tiles, for which each group
//                receives the other's tile maxima through a shared-memory mailbox; one atomicOr
//                per flagged (query tile, key tile); exp2 (a quarter on the FMA pipe); P (bf16)
//                back into TMEM over the consumed S columns; O rescale when the group's reference
//                max grew by more than 2^8.
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
  const int32_t* order;     // [B*H*Tq] work order (null: identity)
  int32_t* work_counter;    // zero before launch; null = static striding over items
  int* status;              // device status word
  int B, H;
  int Nq, Nk;               // query / key tokens (equal for self attention)
  int Tq, Tk, W;            // query tiles, key tiles, mask words per query tile (ceil(Tk / 32))
  int n_items;              // B * H * Tq
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
  static constexpr int BM = 128;                 // MMA M = TMEM lanes = query rows of the tile slot
  static constexpr int BQ = BN;                  // valid query rows per query tile
  static constexpr int KST = 2;                  // K stages
  static constexpr int VST = 3;                  // V stages
  static constexpr int THREADS = 320;            // producer warp, MMA warp, 2 softmax warpgroups
  static constexpr int NCHUNK = D / 64;          // 128-byte swizzle atoms along d
  static constexpr int Q_CHUNK = BM * 128;       // bytes between d-chunks of Q in smem
  static constexpr int KV_CHUNK = BN * 128;      // bytes between d-chunks of a K or V tile
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr uint32_t Q_TX = BQ * D * 2;   // bytes the Q load delivers
  static constexpr uint32_t KV_TX = BN * D * 2;  // bytes of one K or V tile
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_CTL = OFF_V + VST * KV_BYTES;
  static constexpr int CTL_BYTES = 512;
  static constexpr int OFF_X = OFF_CTL + CTL_BYTES;  // tile-max mailbox float[4][128]; epilogue float[2][2][128]
  static constexpr int X_BYTES = 4 * 128 * 4 + 2 * 2 * 128 * 4;
  // O staging for the TMA stores of the epilogue: per softmax warp, 16 rows of its group's D/2
  // columns (D bytes a row; 128-byte swizzled for D = 128, so the region is 1024-aligned)
  static constexpr int OST_ROWS = 16;
  static constexpr int OST_WARP = OST_ROWS * D;
  static constexpr int OFF_OST = (OFF_X + X_BYTES + 1023) / 1024 * 1024;
  static constexpr int OST_BYTES = 8 * OST_WARP;
  // one CTA per SM: the request is padded so that two never fit (TMEM is sized for one)
  static constexpr int SMEM_USED = OFF_OST + OST_BYTES + 1024;
  static constexpr int SMEM_BYTES = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  // TMEM columns: S_0 [0, BN), S_1 [BN, 2BN), O_0 [2BN, 2BN+D), O_1 [2BN+D, 2BN+2D)
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t O_COL = 2 * BN;
  static constexpr uint32_t TMEM_COLS = (2 * BN + 2 * D) <= 256 ? 256 : 512;
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

// A work item (one query tile of one head), decoded once by the producer and handed to the other
// roles through shared memory, with its first two list entries (the first tile of each group).
struct ItemInfo {
  int row;     // (b*H + h)*Tq + qi; -1 marks the end of the work
  int n;       // live key tiles
  int b, h, qi;
  int e0, e1;  // list entries 0 and 1 (when n > 0, n > 1)
};

// Control block in shared memory (barriers are 8-byte mbarrier objects).
struct alignas(8) AttnCtl {
  uint64_t q_full, q_empty;
  uint64_t kv_full[2];               // load bundle t landed: K_t (stage t%2) and V_{t-1} (stage (t-1)%3)
  uint64_t s_full[2];                // S_t ready (buffer t%2, one warpgroup each)
  uint64_t p_full[2];                // P_t written (buffer t%2)
  uint64_t pv_done[2];               // last PV of group g in an item finished (accumulator g)
  uint64_t mx_full[4], mx_empty[4];  // row maxima of tile t posted in / read from mailbox slot t%4
  uint64_t o_free;                   // epilogue has read both O accumulators
  uint64_t item_full[2], item_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  ItemInfo info[2];                  // the handed-out items
  int abort;
  uint32_t tiles;                    // live tiles this CTA processed (measurement hook)
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
  __device__ __forceinline__ void give_up() const {
    *abort = 1;
    atomicCAS(status, 0, kStatusTimeout);
    __threadfence_block();
  }
};

__device__ __forceinline__ int key_entry(const AttnParams& p, int row, int idx);

__device__ __forceinline__ ItemInfo decode_item(const AttnParams& p, int item) {
  ItemInfo it;
  it.row = p.order ? p.order[item] : item;
  it.n = p.counts ? p.counts[it.row] : p.Tk;
  const int bh = it.row / p.Tq;
  it.qi = it.row - bh * p.Tq;
  it.b = bh / p.H;
  it.h = bh - it.b * p.H;
  it.e0 = it.n > 0 ? key_entry(p, it.row, 0) : 0;
  it.e1 = it.n > 1 ? key_entry(p, it.row, 1) : 0;
  return it;
}

// idx-th live key tile of a row, with its kListNoFlag tag (dense: Tk-1, Tk-2, ..., untagged)
__device__ __forceinline__ int key_entry(const AttnParams& p, int row, int idx) {
  return p.list ? int(p.list[size_t(row) * p.Tk + idx]) : (p.Tk - 1 - idx);
}

template <int D, int BN>
__global__ void __launch_bounds__(320, 1)
    lite_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                     const AttnParams p) {
  using C = AttnCfg<D, BN>;
  static_assert(sizeof(AttnCtl) <= C::CTL_BYTES, "control block");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnCtl* ctl = reinterpret_cast<AttnCtl*>(smem + C::OFF_CTL);
  float* mailbox = reinterpret_cast<float*>(smem + C::OFF_X);    // [4][128] tile row maxima
  float* epi = mailbox + 4 * 128;                                // [2 groups][2 values][128]
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
      ptx::mbar_init(BAR(s_full[b]), 1);
      ptx::mbar_init(BAR(p_full[b]), 128);
      ptx::mbar_init(BAR(pv_done[b]), 1);
      ptx::mbar_init(BAR(item_full[b]), 1);
      ptx::mbar_init(BAR(item_empty[b]), 9);  // MMA thread + one lane of each softmax warp
    }
    for (int b = 0; b < 4; ++b) {
      ptx::mbar_init(BAR(mx_full[b]), 128);
      ptx::mbar_init(BAR(mx_empty[b]), 128);
    }
    ptx::mbar_init(BAR(o_free), 256);
    ptx::mbar_init(BAR(drain), 1);
    ctl->abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    ptx::prefetch_tmap(&tmO);
  }
  if constexpr (C::BQ < C::BM) {
    // Q rows past the query tile are never loaded; keep them zero so their S rows stay finite.
    for (int c = 0; c < C::NCHUNK; ++c) {
      uint4* z = reinterpret_cast<uint4*>(smem + C::OFF_Q + c * C::Q_CHUNK + C::BQ * 128);
      for (int x = threadIdx.x; x < (C::BM - C::BQ) * 128 / 16; x += blockDim.x) z[x] = make_uint4(0, 0, 0, 0);
    }
    ptx::fence_proxy_async_smem();
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

  // Barrier phases: t counts the live tiles of all items this CTA processes, in processing order.
  // Tile t uses S buffer, P slot, accumulator and softmax warpgroup t%2, K stage t%2, V stage t%3,
  // mailbox slot t%4. Every waiter either observes each phase of a barrier in order, or is
  // guaranteed by the order of the MMA thread's commits that the barrier is at most one phase
  // away from the awaited one, so the parity waits are exact.
  if (warp == 0) {
    // ------------------------------------------------------------------------- TMA producer
    // Load bundle t carries K_t (stage t%2, last read by QK_{t-2}) and V_{t-1} (stage (t-1)%3, last
    // read by PV_{t-4}, which the MMA thread issues before QK_{t-2}); one wait for QK_{t-2} frees
    // both, and the MMA thread waits once per tile for the bundle. Bundles follow the CTA's tile
    // sequence across items; one last bundle carries only the final V.
    if (lane == 0) {
      uint32_t t = 0, items = 0, qn = 0;
      bool ok = true;
      // last armed phase of each full barrier, so that every issued load can be drained at exit
      bool q_armed = false, kv_armed[2] = {false, false};
      uint32_t q_par = 0, kv_par[2] = {0, 0};
      int pj = 0, ph = 0, pb = 0;  // coordinates of tile t-1
      // s_full of buffer t%2 next completes with QK_t, which needs this bundle: the wait is exact
      auto bundle = [&](bool with_k, int j, int h, int b) -> bool {
        LITE_TRACE(0, 0, t);
        if (t >= 2 && !wt.wait(BAR(s_full[t & 1]), ((t - 2) >> 1) & 1)) return false;
        const uint32_t bar = BAR(kv_full[t & 1]);
        ptx::mbar_arrive_expect_tx(bar, (with_k ? C::KV_TX : 0u) + (t >= 1 ? C::KV_TX : 0u));
        if (with_k) ptx::tma_load_5d(sK + (t & 1) * C::KV_BYTES, &tmK, bar, 0, j * BN, 0, h, b);
        if (t >= 1) ptx::tma_load_5d(sV + ((t - 1) % 3) * C::KV_BYTES, &tmV, bar, 0, pj * BN, 0, ph, pb);
        kv_armed[t & 1] = true;
        kv_par[t & 1] = (t >> 1) & 1;
        LITE_TRACE(0, 1, t);
        pj = j;
        ph = h;
        pb = b;
        ++t;
        return true;
      };
      while (ok) {
        const int slot = items & 1;
        if (items >= 2) ok = wt.wait(BAR(item_empty[slot]), ((items >> 1) - 1) & 1);
        if (!ok) break;
        // dynamic hand-out in schedule order; without a counter, static striding (uniform items)
        int item = p.work_counter ? atomicAdd(p.work_counter, 1) : int(blockIdx.x + items * gridDim.x);
        if (item >= p.n_items) item = -1;
        ItemInfo it{-1, 0, 0, 0, 0, 0, 0};
        if (item >= 0) it = decode_item(p, item);
        ctl->info[slot] = it;
        ptx::mbar_arrive(BAR(item_full[slot]));
        ++items;
        if (item < 0) break;
        if (it.n == 0) continue;
        // Q is read by one item's QKs; q_empty is committed after the item's last QK
        if (qn >= 1) ok = wt.wait(BAR(q_empty), (qn - 1) & 1);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(BAR(q_full), C::Q_TX);
        ptx::tma_load_5d(sQ, &tmQ, BAR(q_full), 0, it.qi * C::BQ, 0, it.h, it.b);
        q_armed = true;
        q_par = qn & 1;
        ++qn;
        for (int idx = 0; idx < it.n && ok; ++idx)
          ok = bundle(true, (idx == 0 ? it.e0 : idx == 1 ? it.e1 : key_entry(p, it.row, idx)) & kListIndexMask,
                      it.h, it.b);
      }
      ctl->tiles = t;
      if (ok && t >= 1) bundle(false, 0, 0, 0);  // V of the last tile
      // Drain: every issued TMA load has landed before this thread leaves (no other thread arms these
      // barriers, so the last armed phase is the one to wait for).
      if (q_armed) wt.wait_drain(BAR(q_full), q_par);
      for (int b = 0; b < 2; ++b)
        if (kv_armed[b]) wt.wait_drain(BAR(kv_full[b]), kv_par[b]);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------------- MMA issuer
    // One thread issues, over the CTA's tile sequence (continuously across items):
    //   QK_t:      S_{t%2} = Q K_t^T          after load bundle t (K_t, V_{t-1}) landed
    //   PV_{t-1}:  O_{(t-1)%2} += P_{t-1} V_{t-1}   after the softmax released P_{t-1}
    // Per tile that is two waits, two fences and one commit; the softmax releases P well ahead of
    // this point, so the waits rarely block. QK_{t+2} reuses S buffer t%2 after PV_t read P_t from
    // it: MMAs of this thread run in issue order.
    if (lane == 0) {
      uint32_t t = 0, items = 0, qn = 0;
      bool ok = true;
      bool stalled = false;
      // the tile whose PV is pending: its item number, index in the item and the item's tile count
      uint32_t pend_item = 0;
      int pend_idx = 0, pend_n = 0;
      // 128B-swizzled K-major operands advance 32 bytes (>> 4 = 2) per K=16 step inside an atom;
      // V (MN-major) advances 16 rows = 2048 bytes (>> 4 = 128) per step.
      const uint64_t q_desc = umma_desc_sw128(sQ, 16, 1024);
      const uint64_t k_desc0 = umma_desc_sw128(sK, 16, 1024);
      const uint64_t v_desc0 = umma_desc_sw128(sV, C::KV_CHUNK, 1024);
      // shared-memory addresses of the per-buffer barriers (8 bytes apart), computed once
      const uint32_t bar_kv = BAR(kv_full[0]), bar_s = BAR(s_full[0]);
      const uint32_t bar_p = BAR(p_full[0]), bar_pv = BAR(pv_done[0]);
      uint32_t v_stage = 0;  // (t-1) % 3 for the pending PV
      auto issue_pv = [&](uint32_t u) -> bool {
        // the first PV of an item overwrites O_0 / O_1 (the first two, one per accumulator): the
        // previous item's epilogue must have read both (o_free: one phase per item, exact because
        // the next phase needs this item's PVs)
        if (pend_idx == 0 && pend_item >= 1 && !wt.wait(BAR(o_free), (pend_item - 1) & 1)) return false;
        LITE_TRACE(1, 3, u);
        // p_full of buffer u%2 next completes for tile u+2, whose S needs QK_{u+2}, issued after this
        if (!wt.wait(bar_p + (u & 1) * 8, (u >> 1) & 1)) return false;
        LITE_TRACE(1, 4, u);
        ptx::tc_fence_after();
        const uint32_t p_tmem = tmem + C::S_COL + (u & 1) * BN;
        const uint32_t o_tmem = tmem + C::O_COL + (u & 1) * D;
        const uint64_t vd = v_desc0 + uint64_t(v_stage * (C::KV_BYTES >> 4));
        v_stage = v_stage == 2 ? 0 : v_stage + 1;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk)
          ptx::mma_ts(o_tmem, p_tmem + kk * 8, vd + uint64_t(kk * 128), C::IDESC_PV,
                      (pend_idx < 2 && kk == 0) ? 0u : 1u);
        // the epilogue of group u%2 waits for the item's last PV into its accumulator
        if (pend_idx >= pend_n - 2) ptx::mma_commit(bar_pv + (u & 1) * 8);
        LITE_TRACE(1, 6, u);
        return true;
      };
      while (ok) {
        const int slot = items & 1;
        ok = wt.wait(BAR(item_full[slot]), (items >> 1) & 1);
        if (!ok) break;
        const ItemInfo it = ctl->info[slot];
        ptx::mbar_arrive(BAR(item_empty[slot]));
        ++items;
        if (it.row < 0) break;
        if (it.n == 0) continue;
        if (p.debug_stall && !stalled) {
          // test hook: withhold all work of this item until the softmax warps give up
          stalled = true;
          const uint64_t s0 = ptx::globaltimer();
          while (!ctl->abort && ptx::globaltimer() - s0 < 4ull * p.wait_limit_ns) {
          }
          if (!ctl->abort) wt.give_up();
          ok = false;
          break;
        }
        // q_full completes once per item; the next load waits for this item's q_empty commit
        ok = wt.wait(BAR(q_full), qn & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        for (int idx = 0; idx < it.n && ok; ++idx, ++t) {
          // kv_full of this slot next completes for bundle t+2, loaded after QK_t finished
          LITE_TRACE(1, 0, t);
          if (!wt.wait(bar_kv + (t & 1) * 8, (t >> 1) & 1)) { ok = false; break; }
          LITE_TRACE(1, 1, t);
          ptx::tc_fence_after();
          const uint64_t kd = k_desc0 + uint64_t(((t & 1) * C::KV_BYTES) >> 4);
          const uint32_t s_tmem = tmem + C::S_COL + (t & 1) * BN;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t off = uint64_t((kk >> 2) * (C::Q_CHUNK >> 4) + (kk & 3) * 2);
            const uint64_t offk = uint64_t((kk >> 2) * (C::KV_CHUNK >> 4) + (kk & 3) * 2);
            ptx::mma_ss(s_tmem, q_desc + off, kd + offk, C::IDESC_QK, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(bar_s + (t & 1) * 8);
          if (idx == it.n - 1) ptx::mma_commit(BAR(q_empty));
          LITE_TRACE(1, 2, t);
          if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
          pend_item = qn;
          pend_idx = idx;
          pend_n = it.n;
        }
        ++qn;
      }
      // the last tile's PV, once the final bundle (its V) has landed
      if (ok && t >= 1) {
        ok = wt.wait(BAR(kv_full[t & 1]), (t >> 1) & 1);
        if (ok) {
          ptx::tc_fence_after();
          issue_pv(t - 1);
        }
      }
      // all issued tensor-core work must finish before TMEM is released
      ptx::mma_commit(BAR(drain));
      wt.wait_drain(BAR(drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------- softmax warpgroups
    const int grp = (warp - 2) >> 2;                // tiles t with t % 2 == grp
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;              // TMEM lane = row inside the tile slot
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    const uint32_t vote_bar = 1 + grp;              // named barrier of this warpgroup (128 threads)
    uint32_t t0 = 0, items = 0, pv_phase = 0;
    while (true) {
      const int slot = items & 1;
      bool ok = wt.wait(BAR(item_full[slot]), (items >> 1) & 1);
      const ItemInfo it = ctl->info[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(BAR(item_empty[slot]));
      ++items;
      if (!ptx::named_bar_and(3, 256, ok) || it.row < 0) break;
      const int n_row = it.qi * C::BQ + r;
      const bool valid_row = (r < C::BQ) && (n_row < p.Nq);
      const size_t o_off = (size_t(it.b) * p.Nq + n_row) * p.H + it.h;
      if (it.n == 0) {
        if (valid_row) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + o_off * D + grp * (D / 2));
          for (int x = 0; x < D / 16; ++x) dst[x] = make_uint4(0, 0, 0, 0);
          if (p.lse && grp == 0) p.lse[(size_t(it.b) * p.H + it.h) * p.Nq + n_row] = -INFINITY;
        }
        continue;
      }
      float m_true = -INFINITY;  // running max over all earlier tiles of the item (log2 units)
      float m_used = -INFINITY;  // this group's exponent reference (lazy rescale)
      float l = 0.f;             // this group's share of the row sum
      // this group's tiles of the item: idx = first, first + 2, ...
      const int first = int((uint32_t(grp) - t0) & 1u);
      int j_next = first < it.n ? (first == 0 ? it.e0 : it.e1) : 0;
      for (int idx = first; idx < it.n; idx += 2) {
        const uint32_t t = t0 + idx;
        const int j = j_next & kListIndexMask;
        const bool may_flag = !(j_next & kListNoFlag);
        if (idx + 2 < it.n) j_next = key_entry(p, it.row, idx + 2);  // prefetch
        if (r == 0) LITE_TRACE(2 + grp, 0, t);
        wt.wait(BAR(s_full[grp]), (t >> 1) & 1);
        __syncwarp();
        ptx::tc_fence_after();
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
        const float loc = ptx::fmax3(m0, m1, fmaxf(m2, m3)) * p.scale_log2;
        if (r == 0) LITE_TRACE(2 + grp, 2, t);
        // lazy rescale of this group's accumulator: move the reference only when the tile max
        // exceeds it by more than 8 (log2 units). The previous PV into this accumulator (tile t-2)
        // was issued before QK_t, so it has completed now that S_t is ready; the rescaled O is
        // stored before any P of this tile is released to the MMA thread.
        const bool need = loc > m_used + 8.0f;
        float alpha = 1.f;
        if (need) {
          alpha = ptx::ex2(m_used - loc);
          m_used = loc;
          l *= alpha;
        }
        if (__any_sync(0xffffffffu, need) && idx >= 2) {
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
        // P = 2^(s*scale*log2e - m_used) as bf16 pairs over the S columns (chunk c of 32 key
        // columns -> TMEM columns [16c, 16c+16)), released to the MMA thread in one piece. Packed
        // fp32x2 arithmetic for the affine step and the row sum; one column pair in four is
        // exponentiated on the FMA pipe, the rest on MUFU.
        const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
        const float2 nm2 = make_float2(-m_used, -m_used);
        float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            const float2 a = __ffma2_rn(make_float2(s[32 * c + 2 * x], s[32 * c + 2 * x + 1]), sc2, nm2);
            const float2 pp = ((x & 3) == 3) ? exp2_poly2(a) : make_float2(ptx::ex2(a.x), ptx::ex2(a.y));
            acc[x & 3] = __fadd2_rn(acc[x & 3], pp);
            __nv_bfloat162 h2 = __floats2bfloat162_rn(pp.x, pp.y);
            pk[x] = *reinterpret_cast<uint32_t*>(&h2);
          }
          ptx::tmem_st16(s_tmem + c * 16, pk);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(BAR(p_full[grp]));
        if (r == 0) LITE_TRACE(2 + grp, 6, t);
        // Post this tile's row maxima for the group that takes tile t+1; they enter its QK-Skip
        // running max, which its vote reads after its own P release, so the post is off the path
        // from S to P here too. Slot t%4 is refilled every four tiles, after its reader took tile t-4's.
        if (t >= 4) wt.wait(BAR(mx_empty[t & 3]), ((t >> 2) - 1) & 1);
        mailbox[(t & 3) * 128 + r] = loc;
        ptx::mbar_arrive(BAR(mx_full[t & 3]));
        if (r == 0) LITE_TRACE(2 + grp, 7, t);
        const float2 acc2 = __fadd2_rn(__fadd2_rn(acc[0], acc[1]), __fadd2_rn(acc[2], acc[3]));
        l += acc2.x + acc2.y;
        // QK-Skip vote, off the path from S to P. The running max over the tiles visited before t
        // takes in tile t-1's maxima from the other group; every posted slot is consumed (also at
        // the first tile of an item, where the value is not used) so that the slots stay in step.
        if (t >= 1) {
          wt.wait(BAR(mx_full[(t - 1) & 3]), ((t - 1) >> 2) & 1);
          const float prev = mailbox[((t - 1) & 3) * 128 + r];
          ptx::mbar_arrive(BAR(mx_empty[(t - 1) & 3]));
          if (idx > 0) m_true = fmaxf(m_true, prev);
        }
        if (r == 0) LITE_TRACE(2 + grp, 3, t);
        if (p.skip_test) {
          // QK-Skip: flag tile j when loc - m < tau for every valid row (m over earlier tiles)
          const bool pred = !valid_row || (loc - m_true < p.tau_log2);
          const bool flag = ptx::named_bar_and(vote_bar, 128, pred);
          if (flag && may_flag && r == 0 && p.mask_out && !ctl->abort)
            atomicOr(p.mask_out + size_t(it.row) * p.W + (j >> 5), 1u << (j & 31));
        }
        if (r == 0) LITE_TRACE(2 + grp, 4, t);
        m_true = fmaxf(m_true, loc);
      }
      // epilogue: each group waits for its last PV, the two partial softmaxes are combined,
      // group g writes columns [g*D/2, (g+1)*D/2) of O (bf16, through shared memory and TMA
      // stores) and group 0 the lse
      if (first < it.n) {
        wt.wait(BAR(pv_done[grp]), pv_phase & 1);  // one phase per item in which this group has a tile
        ++pv_phase;
      }
      epi[(grp * 2 + 0) * 128 + r] = m_used;
      epi[(grp * 2 + 1) * 128 + r] = l;
      ptx::tc_fence_before();
      ptx::named_bar_sync(3, 256);
      ptx::tc_fence_after();
      const float mu0 = epi[0 * 128 + r], l0 = epi[1 * 128 + r];
      const float mu1 = epi[2 * 128 + r], l1 = epi[3 * 128 + r];
      // group g holds a partial iff it had a tile in this item (both do when n >= 2)
      const bool has0 = ((0u - t0) & 1u) < uint32_t(it.n);
      const bool has1 = ((1u - t0) & 1u) < uint32_t(it.n);
      const float mm = has0 && has1 ? fmaxf(mu0, mu1) : (has0 ? mu0 : mu1);
      const float a0 = has0 ? ptx::ex2(mu0 - mm) : 0.f;
      const float a1 = has1 ? ptx::ex2(mu1 - mm) : 0.f;
      const float lt = a0 * l0 + a1 * l1;
      const float inv_l = 1.f / lt;
      const float w0 = a0 * inv_l, w1 = a1 * inv_l;
      // The group's D/2 columns of O, combined and rounded to bf16, leave through shared memory:
      // each warp stages the rows of lanes 0-15, then those of lanes 16-31, and its lane 0 issues
      // one TMA store per half (rows past Nq are clipped by the TMA unit). The threads never wait
      // for global memory; a staging half is rewritten only after its previous store has read it.
      uint32_t ow[D / 4];  // this row's D/2 bf16 columns, packed in pairs
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        const int col = grp * (D / 2) + c * 32;
        uint32_t r0[32], r1[32];
        ptx::tmem_ld32(tmem + lane_base + C::O_COL + 0 * D + col, r0);
        ptx::tmem_ld32(tmem + lane_base + C::O_COL + 1 * D + col, r1);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 16; ++x) {
          // an accumulator without a partial may hold stale data: select, never multiply by zero
          const float o0 = (has0 ? w0 * __uint_as_float(r0[2 * x]) : 0.f) +
                           (has1 ? w1 * __uint_as_float(r1[2 * x]) : 0.f);
          const float o1 = (has0 ? w0 * __uint_as_float(r0[2 * x + 1]) : 0.f) +
                           (has1 ? w1 * __uint_as_float(r1[2 * x + 1]) : 0.f);
          __nv_bfloat162 h2 = __floats2bfloat162_rn(o0, o1);
          ow[c * 16 + x] = *reinterpret_cast<uint32_t*>(&h2);
        }
      }
      {
        uint8_t* stage = smem + C::OFF_OST + (grp * 4 + quarter) * C::OST_WARP;
        const int srow = lane & (C::OST_ROWS - 1);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (lane == 0) ptx::bulk_wait_group_read0();
          __syncwarp();
          if ((lane >> 4) == half) {
#pragma unroll
            for (int x = 0; x < D / 16; ++x) {
              // 16-byte chunk x of the row; 128-byte swizzle (chunk ^ row % 8) for D = 128
              const int pc = D == 128 ? (x ^ (srow & 7)) : x;
              *reinterpret_cast<uint4*>(stage + srow * D + pc * 16) =
                  make_uint4(ow[4 * x], ow[4 * x + 1], ow[4 * x + 2], ow[4 * x + 3]);
            }
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          const int row_in_tile = quarter * 32 + half * C::OST_ROWS;
          if (lane == 0 && row_in_tile < C::BQ && it.qi * C::BQ + row_in_tile < p.Nq) {
            ptx::tma_store_5d(&tmO, ptx::smem_addr(stage), grp * (D / 2) % 64, it.qi * C::BQ + row_in_tile,
                              grp * (D / 2) / 64, it.h, it.b);
            ptx::bulk_commit_group();
          }
        }
      }
      if (valid_row && grp == 0 && p.lse)
        p.lse[(size_t(it.b) * p.H + it.h) * p.Nq + n_row] = (mm + __log2f(lt)) * 0.6931471805599453f;
      ptx::tc_fence_before();
      ptx::mbar_arrive(BAR(o_free));
      t0 += it.n;
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
