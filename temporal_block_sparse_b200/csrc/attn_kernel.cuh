// attn_kernel.cuh -- persistent block-sparse attention forward for sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA per SM walks a list of work items; an item is one query tile of one (b, h). For an item
// it streams only the live key tiles of that query tile (LiteAttention README, "Full-Stage
// Elimination": a skipped tile costs no K/V load, no QK^T, no softmax, no PV), from the highest
// key-tile index down (README, must_do_list: "we iterate in reverse order inside of the kernel").
//
// Warp roles (192 threads):
//   warp 0       TMA producer: Q once per item, then K_j and V_j per live tile into a 2-stage ring.
//   warp 1       TMEM allocator and single-thread tcgen05 MMA issuer:
//                  S_j = Q K_j^T  (SS form, fp32 accumulators in TMEM, double buffered),
//                  O  += P_j V_j  (TS form: P read from TMEM, V from shared memory).
//   warps 2..5   softmax: one thread per query row (TMEM lane). Per tile: row max, the QK-Skip
//                vote (skill page "Lite Attention Temporal Sparse", Core Concept: a tile whose local
//                max score is far below the cumulative max is flagged), one atomicOr per flagged
//                (query tile, key tile), exp2, row sum, P (bf16) back to TMEM, O rescale when the
//                running max moved by more than 2^8; epilogue O / l and lse.
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

struct AttnParams {
  __nv_bfloat16* o;         // [B, N, H, D]
  float* lse;               // [B, H, N] or null
  uint32_t* mask_out;       // [B, H, T, W] or null (flags not recorded)
  const int16_t* list;      // [B*H*T, T] live key tiles, descending (null: all tiles, dense)
  const int32_t* counts;    // [B*H*T] live counts (null: T each)
  const int32_t* order;     // [B*H*T] work order (null: identity)
  int32_t* work_counter;    // zero before launch; null = static striding over items
  int* status;              // device status word
  int B, H, N, T, W;
  int n_items;
  float scale_log2;         // softmax scale * log2(e)
  float tau_log2;           // QK-Skip threshold * log2(e)
  int skip_test;            // 1: run the QK-Skip vote and record flags
  unsigned long long wait_limit_ns;
  int debug_stall;          // test hook: MMA warp withholds its first tile
};

template <int D, int BN>
struct AttnCfg {
  static constexpr int BM = 128;                 // MMA M = TMEM lanes = query rows of the tile slot
  static constexpr int BQ = BN;                  // valid query rows per query tile
  static constexpr int STAGES = 2;               // K/V ring depth
  static constexpr int NCHUNK = D / 64;          // 128-byte swizzle atoms along d
  static constexpr int Q_CHUNK = BM * 128;       // bytes between d-chunks of Q in smem
  static constexpr int KV_CHUNK = BN * 128;      // bytes between d-chunks of a K or V tile
  static constexpr int Q_BYTES = BM * D * 2;
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr uint32_t Q_TX = BQ * D * 2;   // bytes the Q load delivers
  static constexpr uint32_t KV_TX = BN * D * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;
  static constexpr int OFF_V = OFF_K + STAGES * KV_BYTES;
  static constexpr int OFF_CTL = OFF_V + STAGES * KV_BYTES;
  static constexpr int CTL_BYTES = 512;
  // one CTA per SM: the request is padded so that two never fit (TMEM is sized for one)
  static constexpr int SMEM_USED = OFF_CTL + CTL_BYTES + 1024;
  static constexpr int SMEM_BYTES = SMEM_USED > 120 * 1024 ? SMEM_USED : 120 * 1024;
  // TMEM columns: S buffers at [0, BN) and [BN, 2BN); O at [2BN, 2BN + D)
  static constexpr uint32_t S_COL = 0;
  static constexpr uint32_t O_COL = 2 * BN;
  static constexpr uint32_t TMEM_COLS = (2 * BN + D) <= 256 ? 256 : 512;
  // instruction descriptors, kind::f16: fp32 accumulate (bit 4), bf16 A (bits 7-9) and B (10-12),
  // B major-ness (bit 16), N >> 3 (bits 17-22), M >> 4 (bits 24-28)
  static constexpr uint32_t IDESC_QK = (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(BN >> 3) << 17) |
                                       (uint32_t(BM >> 4) << 24);
  static constexpr uint32_t IDESC_PV = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 16) |
                                       (uint32_t(D >> 3) << 17) | (uint32_t(BM >> 4) << 24);
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(BN == 64 || BN == 128, "tile");
  static_assert(2 * BN + D <= 512, "TMEM budget");
};

// Control block in shared memory (barriers are 8-byte mbarrier objects).
struct alignas(8) AttnCtl {
  uint64_t q_full, q_empty;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], p_full[2];
  uint64_t pv_done, o_free;
  uint64_t item_full[2], item_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int item[2];
  int abort;
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

struct ItemInfo {
  int row;  // (b*H + h)*T + qi
  int n;    // live key tiles
  int b, h, qi;
};

__device__ __forceinline__ ItemInfo decode_item(const AttnParams& p, int item) {
  ItemInfo it;
  it.row = p.order ? p.order[item] : item;
  it.n = p.counts ? p.counts[it.row] : p.T;
  const int bh = it.row / p.T;
  it.qi = it.row - bh * p.T;
  it.b = bh / p.H;
  it.h = bh - it.b * p.H;
  return it;
}

__device__ __forceinline__ int key_tile(const AttnParams& p, int row, int idx) {
  return p.list ? int(p.list[size_t(row) * p.T + idx]) : (p.T - 1 - idx);
}

template <int D, int BN>
__global__ void __launch_bounds__(192, 1)
    lite_attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV, const AttnParams p) {
  using C = AttnCfg<D, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnCtl* ctl = reinterpret_cast<AttnCtl*>(smem + C::OFF_CTL);
  const uint32_t sQ = ptx::smem_addr(smem + C::OFF_Q);
  const uint32_t sK = ptx::smem_addr(smem + C::OFF_K);
  const uint32_t sV = ptx::smem_addr(smem + C::OFF_V);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

#define BAR(x) ptx::smem_addr(&ctl->x)

  if (threadIdx.x == 0) {
    ptx::mbar_init(BAR(q_full), 1);
    ptx::mbar_init(BAR(q_empty), 1);
    for (int s = 0; s < 2; ++s) {
      ptx::mbar_init(BAR(k_full[s]), 1);
      ptx::mbar_init(BAR(k_empty[s]), 1);
      ptx::mbar_init(BAR(v_full[s]), 1);
      ptx::mbar_init(BAR(v_empty[s]), 1);
      ptx::mbar_init(BAR(s_full[s]), 1);
      ptx::mbar_init(BAR(p_full[s]), 128);
      ptx::mbar_init(BAR(item_full[s]), 1);
      ptx::mbar_init(BAR(item_empty[s]), 5);  // MMA thread + one lane of each softmax warp
    }
    ptx::mbar_init(BAR(pv_done), 1);
    ptx::mbar_init(BAR(o_free), 128);
    ptx::mbar_init(BAR(drain), 1);
    ctl->abort = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
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

  if (warp == 0) {
    // ------------------------------------------------------------------------- TMA producer
    if (lane == 0) {
      uint32_t kv = 0, items = 0, qn = 0;
      bool ok = true;
      // last armed phase of each full barrier, so that every issued load can be drained at exit
      bool q_armed = false, k_armed[2] = {false, false}, v_armed[2] = {false, false};
      uint32_t q_par = 0, k_par[2] = {0, 0}, v_par[2] = {0, 0};
      while (ok) {
        const int slot = items & 1;
        if (items >= 2) ok = wt.wait(BAR(item_empty[slot]), ((items >> 1) - 1) & 1);
        if (!ok) break;
        // dynamic hand-out in schedule order; without a counter, static striding (uniform items)
        int item = p.work_counter ? atomicAdd(p.work_counter, 1) : int(blockIdx.x + items * gridDim.x);
        if (item >= p.n_items) item = -1;
        ctl->item[slot] = item;
        ptx::mbar_arrive(BAR(item_full[slot]));
        ++items;
        if (item < 0) break;
        const ItemInfo it = decode_item(p, item);
        if (it.n == 0) continue;
        if (qn >= 1) ok = wt.wait(BAR(q_empty), (qn - 1) & 1);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(BAR(q_full), C::Q_TX);
        for (int c = 0; c < C::NCHUNK; ++c)
          ptx::tma_load_4d(sQ + c * C::Q_CHUNK, &tmQ, BAR(q_full), c * 64, it.h, it.qi * C::BQ, it.b);
        q_armed = true;
        q_par = qn & 1;
        ++qn;
        for (int idx = 0; idx < it.n && ok; ++idx, ++kv) {
          const int j = key_tile(p, it.row, idx);
          const int s = kv & 1;
          const uint32_t ph = (kv >> 1) & 1;
          if (kv >= 2) ok = wt.wait(BAR(k_empty[s]), ph ^ 1);
          if (!ok) break;
          ptx::mbar_arrive_expect_tx(BAR(k_full[s]), C::KV_TX);
          for (int c = 0; c < C::NCHUNK; ++c)
            ptx::tma_load_4d(sK + s * C::KV_BYTES + c * C::KV_CHUNK, &tmK, BAR(k_full[s]), c * 64, it.h,
                             j * BN, it.b);
          k_armed[s] = true;
          k_par[s] = ph;
          if (kv >= 2) ok = wt.wait(BAR(v_empty[s]), ph ^ 1);
          if (!ok) break;
          ptx::mbar_arrive_expect_tx(BAR(v_full[s]), C::KV_TX);
          for (int c = 0; c < C::NCHUNK; ++c)
            ptx::tma_load_4d(sV + s * C::KV_BYTES + c * C::KV_CHUNK, &tmV, BAR(v_full[s]), c * 64, it.h,
                             j * BN, it.b);
          v_armed[s] = true;
          v_par[s] = ph;
        }
      }
      // Drain: every issued TMA load has landed before this thread leaves (no other thread arms these
      // barriers, so the last armed phase is the one to wait for).
      if (q_armed) wt.wait_drain(BAR(q_full), q_par);
      for (int s = 0; s < 2; ++s) {
        if (k_armed[s]) wt.wait_drain(BAR(k_full[s]), k_par[s]);
        if (v_armed[s]) wt.wait_drain(BAR(v_full[s]), v_par[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      uint32_t kv = 0, g = 0, items = 0, qn = 0;
      bool ok = true;
      bool stalled = false;
      auto issue_pv = [&](uint32_t gi, uint32_t kvi, bool first_of_item) -> bool {
        const uint32_t buf = gi & 1;
        const uint32_t s = kvi & 1;
        if (!wt.wait(BAR(p_full[buf]), (gi >> 1) & 1)) return false;
        if (!wt.wait(BAR(v_full[s]), (kvi >> 1) & 1)) return false;
        ptx::tc_fence_after();
        const uint32_t p_tmem = tmem + C::S_COL + buf * BN;
        const uint32_t v_base = sV + s * C::KV_BYTES;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          const uint64_t bdesc = umma_desc_sw128(v_base + kk * 2048, C::KV_CHUNK, 1024);
          ptx::mma_ts(tmem + C::O_COL, p_tmem + kk * 8, bdesc, C::IDESC_PV, (first_of_item && kk == 0) ? 0u : 1u);
        }
        ptx::mma_commit(BAR(pv_done));
        ptx::mma_commit(BAR(v_empty[s]));
        return true;
      };
      while (ok) {
        const int slot = items & 1;
        ok = wt.wait(BAR(item_full[slot]), (items >> 1) & 1);
        if (!ok) break;
        const int item = ctl->item[slot];
        ptx::mbar_arrive(BAR(item_empty[slot]));
        ++items;
        if (item < 0) break;
        const ItemInfo it = decode_item(p, item);
        if (it.n == 0) continue;
        if (p.debug_stall && !stalled) {
          // test hook: withhold all work of this item until the softmax warps give up
          stalled = true;
          const uint64_t t0 = ptx::globaltimer();
          while (!ctl->abort && ptx::globaltimer() - t0 < 4ull * p.wait_limit_ns) {
          }
          if (!ctl->abort) wt.give_up();
          ok = false;
          break;
        }
        ok = wt.wait(BAR(q_full), qn & 1);
        if (!ok) break;
        ptx::tc_fence_after();
        for (int idx = 0; idx < it.n && ok; ++idx) {
          const uint32_t gi = g + idx, kvi = kv + idx;
          const uint32_t buf = gi & 1, s = kvi & 1;
          ok = wt.wait(BAR(k_full[s]), (kvi >> 1) & 1);
          if (!ok) break;
          ptx::tc_fence_after();
          const uint32_t k_base = sK + s * C::KV_BYTES;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk & 3) * 32;  // 16 bf16 = 32 bytes inside the 128-byte swizzle atom
            const uint64_t adesc = umma_desc_sw128(sQ + (kk >> 2) * C::Q_CHUNK + off, 16, 1024);
            const uint64_t bdesc = umma_desc_sw128(k_base + (kk >> 2) * C::KV_CHUNK + off, 16, 1024);
            ptx::mma_ss(tmem + C::S_COL + buf * BN, adesc, bdesc, C::IDESC_QK, kk > 0 ? 1u : 0u);
          }
          ptx::mma_commit(BAR(s_full[buf]));
          ptx::mma_commit(BAR(k_empty[s]));
          if (idx == it.n - 1) ptx::mma_commit(BAR(q_empty));
          if (idx >= 1) {
            if (idx == 1 && qn >= 1) ok = wt.wait(BAR(o_free), (qn - 1) & 1);
            if (ok) ok = issue_pv(gi - 1, kvi - 1, idx == 1);
          }
        }
        if (ok) {
          if (it.n == 1 && qn >= 1) ok = wt.wait(BAR(o_free), (qn - 1) & 1);
          if (ok) ok = issue_pv(g + it.n - 1, kv + it.n - 1, it.n == 1);
        }
        g += it.n;
        kv += it.n;
        ++qn;
      }
      // all issued tensor-core work must finish before TMEM is released
      ptx::mma_commit(BAR(drain));
      wt.wait_drain(BAR(drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------------- softmax warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // TMEM lane = row inside the tile slot
    const uint32_t lane_base = uint32_t(quarter * 32) << 16;
    uint32_t g = 0, items = 0, qn = 0;
    while (true) {
      const int slot = items & 1;
      bool ok = wt.wait(BAR(item_full[slot]), (items >> 1) & 1);
      const int item = ctl->item[slot];
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(BAR(item_empty[slot]));
      ++items;
      if (!ptx::named_bar_and(1, 128, ok) || item < 0) break;
      const ItemInfo it = decode_item(p, item);
      const int n_row = it.qi * C::BQ + r;
      const bool valid_row = (r < C::BQ) && (n_row < p.N);
      const size_t o_off = (size_t(it.b) * p.N + n_row) * p.H + it.h;
      if (it.n == 0) {
        if (valid_row) {
          uint4* dst = reinterpret_cast<uint4*>(p.o + o_off * D);
          for (int x = 0; x < D / 8; ++x) dst[x] = make_uint4(0, 0, 0, 0);
          if (p.lse) p.lse[(size_t(it.b) * p.H + it.h) * p.N + n_row] = -INFINITY;
        }
        continue;
      }
      float m_true = -INFINITY;  // running max of visited tiles (log2 units)
      float m_used = -INFINITY;  // max the exponentials are taken against (lazy rescale)
      float l = 0.f;
      for (int idx = 0; idx < it.n; ++idx) {
        const uint32_t gi = g + idx;
        const uint32_t buf = gi & 1;
        const int j = key_tile(p, it.row, idx);
        wt.wait(BAR(s_full[buf]), (gi >> 1) & 1);
        __syncwarp();
        ptx::tc_fence_after();
        const uint32_t s_tmem = tmem + lane_base + C::S_COL + buf * BN;
        uint32_t sr[BN];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) ptx::tmem_ld32(s_tmem + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
        ptx::tmem_wait_ld();
        float s[BN];
#pragma unroll
        for (int x = 0; x < BN; ++x) s[x] = __uint_as_float(sr[x]);
        const int valid_cols = min(BN, p.N - j * BN);
        if (valid_cols < BN) {
          // key columns past N (zero-filled by TMA) take no part in max, sum or PV
#pragma unroll
          for (int x = 0; x < BN; ++x)
            if (x >= valid_cols) s[x] = -INFINITY;
        }
        float mx = s[0];
#pragma unroll
        for (int x = 1; x < BN; ++x) mx = fmaxf(mx, s[x]);
        const float loc = mx * p.scale_log2;
        if (p.skip_test) {
          // QK-Skip: flag tile j when loc - m < tau for every valid row (m over earlier tiles)
          const bool pred = !valid_row || (loc - m_true < p.tau_log2);
          const bool flag = ptx::named_bar_and(1, 128, pred);
          if (flag && r == 0 && p.mask_out && !ctl->abort)
            atomicOr(p.mask_out + size_t(it.row) * p.W + (j >> 5), 1u << (j & 31));
        }
        m_true = fmaxf(m_true, loc);
        // lazy rescale: move the reference max only when it grew by more than 8 (log2 units)
        const bool need = loc > m_used + 8.0f;
        float alpha = 1.f;
        if (need) {
          alpha = ptx::ex2(m_used - loc);
          m_used = loc;
          l *= alpha;
        }
        const bool warp_need = __any_sync(0xffffffffu, need);
        // P = 2^(s*scale*log2e - m_used), bf16 pairs written over the consumed S columns
        const float neg_m = -m_used;
        float rowsum = 0.f;
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) {
          uint32_t pk[32];
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            const float p0 = ptx::ex2(fmaf(s[c * 64 + 2 * x], p.scale_log2, neg_m));
            const float p1 = ptx::ex2(fmaf(s[c * 64 + 2 * x + 1], p.scale_log2, neg_m));
            rowsum += p0 + p1;
            __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
            pk[x] = *reinterpret_cast<uint32_t*>(&h2);
          }
          ptx::tmem_st32(s_tmem + c * 32, pk);
        }
        l += rowsum;
        if (idx > 0) {
          // Every thread observes each PV completion once, in order, so the parity wait is exact.
          // PV_{gi-1} ran while the exponentials above were computed; O is rescaled only after it.
          wt.wait(BAR(pv_done), (gi - 1) & 1);
          __syncwarp();
          if (warp_need) {
            ptx::tc_fence_after();
            const uint32_t o_tmem = tmem + lane_base + C::O_COL;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t rr[32];
              ptx::tmem_ld32(o_tmem + c * 32, rr);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int x = 0; x < 32; ++x) rr[x] = __float_as_uint(__uint_as_float(rr[x]) * alpha);
              ptx::tmem_st32(o_tmem + c * 32, rr);
            }
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        ptx::mbar_arrive(BAR(p_full[buf]));
      }
      // epilogue: wait for the last PV, normalise, store O (bf16) and lse
      wt.wait(BAR(pv_done), (g + it.n - 1) & 1);
      __syncwarp();
      ptx::tc_fence_after();
      const float inv_l = 1.f / l;
      const uint32_t o_tmem = tmem + lane_base + C::O_COL;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t rr[32];
        ptx::tmem_ld32(o_tmem + c * 32, rr);
        ptx::tmem_wait_ld();
        if (valid_row) {
          uint32_t pk[16];
#pragma unroll
          for (int x = 0; x < 16; ++x) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(rr[2 * x]) * inv_l,
                                                      __uint_as_float(rr[2 * x + 1]) * inv_l);
            pk[x] = *reinterpret_cast<uint32_t*>(&h2);
          }
          uint4* dst = reinterpret_cast<uint4*>(p.o + o_off * D + c * 32);
#pragma unroll
          for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        }
      }
      if (valid_row && p.lse)
        p.lse[(size_t(it.b) * p.H + it.h) * p.N + n_row] = (m_used + __log2f(l)) * 0.6931471805599453f;
      ptx::tc_fence_before();
      ptx::mbar_arrive(BAR(o_free));
      g += it.n;
      ++qn;
    }
  }
#undef BAR

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

}  // namespace lite
