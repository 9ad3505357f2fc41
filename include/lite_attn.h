/*
 * lite_attn.h -- C ABI of the B200 (sm_100a) LiteAttention forward pass.
 *
 * LiteAttention ("LiteAttention: A Temporal Sparse Attention for Diffusion Transformers",
 * arXiv 2511.11062; README of moonmath-ai/LiteAttention) is FlashAttention-style softmax
 * self-attention that reads a persistent per-(batch, head, query tile, key tile) Skip-Mask,
 * bypasses every marked tile completely (no QK^T, no softmax, no PV, no K/V load: README,
 * "Full-Stage Elimination"), and on every tile it does compute evaluates the QK-Skip test inside
 * the online softmax (README, "QK-Skip Algorithm"; skill page "Lite Attention Temporal Sparse",
 * Core Concept). Tiles that pass the test are OR-ed into the mask for the next denoising step,
 * so the mask only grows.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All functions are extern "C", return an int status (LITE_OK = 0, negative = error) and never
 *    throw. Work is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream) and the
 *    call returns after enqueueing; nothing synchronises except lite_get_device_status().
 *  - Every buffer is owned by the caller, who allocates and frees it; the library keeps no state
 *    between calls (one mask pair per attention layer, README: separate instances per layer).
 *    Device pointers must be device-accessible memory of the current device.
 *  - Layouts:
 *      q, k, v, o : bf16 [B, N, H, d], contiguous, 16-byte aligned (cross attention: q and o
 *                   [B, Nq, H, d], k and v [B, Nk, H, d]). The output o viewed as
 *                   [B, N, H*d] is the README's (batch, seq_len, heads*head_dim) return layout.
 *      lse        : fp32 [B, H, N], natural log of the softmax normaliser of each query row.
 *      masks      : uint32 [B, H, T, W]. Bit (j & 31) of word (j >> 5) set = skip key tile j for
 *                   that (b, h, query tile). T = ceil(N / tile), W = ceil(T / 32). Bits at or
 *                   above T in the last word are ignored and written as 0.
 *      tile       : 64 for d = 64, 128 for d = 128 (lite_mask_geometry reports it).
 *  - Argument errors are reported before any CUDA call is made.
 */
#ifndef LITE_ATTN_H
#define LITE_ATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* cudaStream_t without pulling in the CUDA headers. */
typedef struct CUstream_st* lite_stream_t;

enum {
  LITE_OK = 0,
  LITE_ERR_INVALID_ARG = -1, /* NULL required pointer, B/H/N <= 0, NaN tau, tau > 0 outside debug */
  LITE_ERR_UNSUPPORTED = -2, /* d not in {64, 128}, misaligned pointer, T or sizes beyond limits  */
  LITE_ERR_CUDA = -3,        /* a CUDA launch, allocation or query failed                          */
  LITE_ERR_TIMEOUT = -4,     /* device status: a kernel wait exceeded its time limit and gave up   */
  LITE_ERR_CHECK = -5,       /* device status: a kernel found a malformed Skip-List or work order  */
  LITE_ERR_SCRATCH_LIMIT = -6 /* lite_attn_fwd_noalloc: the layer needs more than its fixed scratch  */
};

/*
 * lite_attn_fwd -- one LiteAttention forward for one layer at one denoising step.
 *
 * Computes, for every (b, h) and query row n, o = softmax(scale * q k^T) v over the key tiles that
 * mask_in leaves live (README, "Full-Stage Elimination"), and lse = log-sum-exp of those scores
 * (README: LSE is returned for combining partial attentions). While doing so it runs the QK-Skip
 * test on every computed tile: the key tiles of a query tile are visited from the highest index
 * down (README, must_do_list: the kernel walks key positions in reverse order); with m_r the
 * running row maximum of scale*QK^T over the tiles visited before tile j and loc_r the row maximum
 * inside tile j, tile j is flagged when loc_r - m_r < tau for every valid row r of the query tile.
 * mask_out = mask_in | flags (README, "QK-Skip Algorithm": the number of skipped tiles only grows).
 *
 *  q, k, v    in   device bf16 [B, N, H, d].
 *  o          out  device bf16 [B, N, H, d].
 *  lse        out  device fp32 [B, H, N], or NULL to skip writing it.
 *  mask_in    in   device uint32 [B, H, T, W], or NULL = nothing skipped (fresh state, README
 *                  reset_skip_state()).
 *  mask_out   out  device uint32 [B, H, T, W], or NULL = do not record flags. It may equal
 *                  mask_in (in place); otherwise the library first copies mask_in into it.
 *  B, H, N, d      batch, heads, tokens, head dim (d in {64, 128}); T = ceil(N/tile) <= 4096.
 *  scale           softmax scale; <= 0 or NaN selects 1/sqrt(d) (README's Wan2.1 call omits it).
 *  tau             QK-Skip threshold in natural-log units of scale*QK^T (README: default -10;
 *                  -6, -3, 0 in its examples). -inf disables flagging. tau > 0 is refused unless
 *                  the environment variable LITE_ATTN_DEBUG is set to anything but "FALSE"
 *                  (README: LITE_ATTENTION_DEBUG). NaN is refused.
 *  stream          CUDA stream for all work.
 *
 * A query tile whose live list is empty (only possible with a caller-built mask) yields o = 0 and
 * lse = -inf for its rows. Scratch memory (per-row live lists and the work order) is taken with
 * cudaMallocFromPoolAsync on `stream` from a stream-ordered pool the library creates per device
 * (it retains freed memory for reuse; its peak is the largest scratch of any call) and released
 * with cudaFreeAsync on the same stream.
 * Returns LITE_OK once enqueued; device-side failures are reported by lite_get_device_status().
 */
int lite_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                  const uint32_t* mask_in, uint32_t* mask_out, int B, int H, int N, int d,
                  float scale, float tau, lite_stream_t stream);

/*
 * lite_attn_dense -- the no-skip path (README, enable_skip_optimization: with skipping off the
 * library runs plain FlashAttention-3).
 *
 * Same kernel and layouts as lite_attn_fwd with every tile live and the QK-Skip test off; no mask
 * is read or written and no scratch memory is allocated. lse may be NULL.
 */
int lite_attn_dense(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H,
                    int N, int d, float scale, lite_stream_t stream);

/*
 * lite_mask_to_list -- Skip-Mask to Skip-List compaction (skill page, Architecture Overview: the
 * skip state is a bitmask, or a list where sparsity is high; README: key ranges are walked in
 * reverse order).
 *
 *  mask    in   device uint32 [B, H, T, W], or NULL = nothing skipped.
 *  list    out  device int16 [B, H, T, T]: for each (b, h, query tile) the live key tiles in
 *               descending order in the first counts[...] entries; later entries are untouched.
 *  counts  out  device int32 [B, H, T]: number of live key tiles per query tile.
 *  B, H, N, d   as in lite_attn_fwd (they fix T and W).
 */
int lite_mask_to_list(const uint32_t* mask, int16_t* list, int32_t* counts, int B, int H, int N,
                      int d, lite_stream_t stream);

/*
 * lite_mask_to_ranges -- Skip-Mask to range-encoded Skip-List (skill page, Architecture Overview:
 * a bitmask, or a list where sparsity is high; range pairs as in the README's must_do_list: start
 * inclusive, end exclusive, strictly descending, because key tiles are visited in reverse order).
 *
 * For each (b, h, query tile), every maximal run of live key tiles a..b (a <= b, tile indices)
 * becomes the pair (b, a - 1); pairs are written from the highest run down.
 *
 *  mask    in   device uint32 [B, H, T, W], or NULL = nothing skipped (one run T-1 .. 0).
 *  ranges  out  device int16 [B, H, T, T+1]: the first 2*nruns[...] entries of each row hold
 *               start_0, end_0, start_1, end_1, ... with start_0 > end_0 >= start_1 + 1 > ...;
 *               end may be -1. Later entries are untouched. 2-byte aligned.
 *  nruns   out  device int32 [B, H, T]: number of runs per query tile (0 when all are skipped).
 *  B, H, N, d   as in lite_attn_fwd (they fix T and W).
 */
int lite_mask_to_ranges(const uint32_t* mask, int16_t* ranges, int32_t* nruns, int B, int H, int N,
                        int d, lite_stream_t stream);

/*
 * lite_schedule -- longest-first order of query tiles (no counterpart on the pages). The
 * attention kernel behind lite_attn_fwd takes its work in pairs of query tiles of one head (see
 * LITE_OPT_PAIR_STRIDE) and orders those pairs the same way, by their combined live count.
 *
 * Heads (b, h) are ordered by decreasing total live-tile count (ties: lower b*H+h first); inside a
 * head, query tiles by decreasing live count (ties: lower index first). Writes order[B*H*T] with
 * entries (b*H + h)*T + i: a longest-first list schedule that keeps one head's query tiles
 * together so that concurrently running tiles share K/V in L2.
 *
 *  counts  in   device int32 [B, H, T] (from lite_mask_to_list), each in [0, 4096]. For cross
 *               attention T here is the number of QUERY tiles (rows per head).
 *  order   out  device int32 [B*H*T].
 *  B*H <= 8192 and T <= 4096 (LITE_ERR_UNSUPPORTED otherwise).
 */
int lite_schedule(const int32_t* counts, int32_t* order, int B, int H, int T, lite_stream_t stream);

/* Host only: tile edge, tiles per side and mask words per row for (N, d). For cross attention
 * call it with Nq for the query-tile count and with Nk for the key-tile count and the words. */
int lite_mask_geometry(int N, int d, int* tile, int* T, int* words);

/*
 * lite_get_device_status -- synchronises `stream`, then reads and clears the device status word of
 * the current device. Returns LITE_OK, LITE_ERR_TIMEOUT (a kernel wait gave up after its time
 * limit; that call's outputs are invalid), LITE_ERR_CHECK, or LITE_ERR_CUDA if the stream itself
 * reports an error.
 */
int lite_get_device_status(lite_stream_t stream);

/* Static description of a status code; never NULL. */
const char* lite_status_string(int status);

/*
 * Process-wide options (host state, not thread-safe against concurrent launches):
 *  LITE_OPT_WAIT_LIMIT_NS  upper bound, in nanoseconds, on any single in-kernel wait before the
 *                          kernel gives up and reports LITE_ERR_TIMEOUT (default 4e9; >= 1000).
 *  LITE_OPT_DEBUG_STALL    1 = test hook: the MMA warp of every CTA withholds its first tile, so
 *                          the waits that depend on it run out their limit (no fault, no hang).
 *  LITE_OPT_MAX_CTAS       cap on the persistent grid size (0 = every resident CTA slot: one
 *                          CTA per SM with d = 128, two per SM with d = 64).
 *  LITE_OPT_SCHEDULE       1 (default) = lite_attn_fwd* hand out their work items (pairs of
 *                          query tiles of one head, see LITE_OPT_PAIR_STRIDE) longest first, heads
 *                          kept together, as lite_schedule orders query tiles; 0 = in their
 *                          natural (b, h, pair) order, for measuring what the schedule buys.
 *                          Results are identical either way.
 *  LITE_OPT_PAIR_STRIDE    which query tiles share a CTA (and each key tile that is live for both).
 *                          0 (default) = chosen per call from mask_in: the stride s in [1, 64] whose
 *                          pairs (tile r with tile r + s inside each block of 2s tiles) share the
 *                          most live key tiles, the smaller on ties (1 = tiles 2k and 2k+1; without
 *                          mask_in, and for lite_attn_fwd_list, 1). k >= 1 = that stride. Results
 *                          are identical for every stride: each query tile walks its own list.
 * Returns LITE_ERR_INVALID_ARG for an unknown option or out-of-range value.
 */
enum {
  LITE_OPT_WAIT_LIMIT_NS = 1,
  LITE_OPT_DEBUG_STALL = 2,
  LITE_OPT_MAX_CTAS = 3,
  LITE_OPT_SCHEDULE = 4,
  LITE_OPT_PAIR_STRIDE = 5
};
int lite_set_option(int option, long long value);

/*
 * lite_set_cta_timing -- measurement hook for load balance. While set, every attention kernel
 * launch writes, for each CTA b < capacity, buf[3b] = its start time, buf[3b+1] = its end time
 * (both the GPU's global nanosecond timer) and buf[3b+2] = the number of live (query tile, key tile)
 * pairs it computed.
 * buf is caller-owned device memory of 3 * capacity uint64 values (8-byte aligned), or NULL with
 * capacity 0 to stop. Host state, like lite_set_kernel_events.
 */
int lite_set_cta_timing(void* buf, int capacity);

/*
 * lite_set_kernel_events -- measurement hook. While set, every lite_attn_fwd* / lite_attn_dense*
 * call records `before` immediately before and `after` immediately after its attention kernel, on
 * the call's stream. Both are cudaEvent_t handles owned by the caller; pass NULL, NULL to stop.
 */
int lite_set_kernel_events(void* before, void* after);

/*
 * lite_scratch_pool_bytes -- measurement hook. *reserved = device memory, in bytes, that the
 * library's scratch pool on the current device holds (its stream-ordered pool keeps freed memory
 * for reuse); 0 while no pooled call has run on the device, since the pool is created by the
 * first lite_attn_fwd / lite_attn_fwd_ex call. Makes no allocation. LITE_ERR_INVALID_ARG for a
 * NULL pointer.
 */
int lite_scratch_pool_bytes(long long* reserved);

/*
 * lite_attn_fwd_noalloc -- lite_attn_fwd for callers that must not allocate device memory.
 *
 * The LiteAttention paper and pages have no counterpart to this entry point; it exists for
 * embedding the forward pass where the library may not allocate: a serving runtime that has
 * reserved (nearly) all device memory for its own pool, so any allocation by a library fails or
 * evicts the caller's data, or a latency-critical denoising loop that cannot afford an
 * allocator call (which may block or synchronise) on every layer of every step.
 *
 * Arguments, layouts, semantics and results are exactly those of lite_attn_fwd. The difference is
 * where the per-call scratch (live lists, counts, work order, work counter) lives: in one fixed
 * array of LITE_NOALLOC_SCRATCH_BYTES (8 MiB) that the library defines in device memory. Every GPU
 * that loads the library holds that array until the process exits. This call makes no cudaMalloc,
 * cudaFree or other allocating call, and creates no memory pool (the scratch pool behind
 * lite_attn_fwd is created by the first lite_attn_fwd / lite_attn_fwd_ex call on a device, never
 * by this one; lite_scratch_pool_bytes reports whether it exists).
 *
 *  - Limit: the layer's scratch must fit in 8 MiB. With R = B*H*T and T = ceil(N / tile) it is
 *    up256(2*R*T) + 2*up256(4*R) + 512 bytes (up256 rounds up to a multiple of 256), about
 *    R*(2T + 8). The 480p layer (B=1, H=40, N=32760, d=128: 5.3 MB) fits; the 720p layer
 *    (N=75600: 28 MB) does not. Layers that do not fit return LITE_ERR_SCRATCH_LIMIT before any
 *    work is enqueued.
 *  - Set-up: the first call on each device looks up the array's device address (with that device
 *    current), the device's SM count and the status word's address; make that first call before
 *    capturing any stream into a CUDA graph.
 *  - Sharing: all calls on a device use the same array, and it keeps whatever the last call left
 *    in it (the work counter is cleared on the stream at the start of every call). Calls whose
 *    work overlaps on the GPU -- for example on two streams without ordering between them --
 *    race on the array and give wrong results; order them on one stream or with events.
 */
#define LITE_NOALLOC_SCRATCH_BYTES (8u << 20)
int lite_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                          const uint32_t* mask_in, uint32_t* mask_out, int B, int H, int N, int d,
                          float scale, float tau, lite_stream_t stream);

/*
 * lite_attn_fwd_list -- lite_attn_fwd over caller-supplied Skip-Lists instead of a Skip-Mask.
 *
 * The skill page "Lite Attention Temporal Sparse" (Architecture Overview) keeps the skip state as a
 * bitmask, or as a list where sparsity is high: per (b, h, query tile) the live key tiles, which
 * the kernel visits from the highest index down (README, must_do_list: key positions are walked in
 * reverse order). lite_attn_fwd builds these lists from the mask (lite_mask_to_list) on every
 * call; a caller that keeps the lists itself passes them here, and the compaction step and the mask
 * copy are skipped. Results are those of lite_attn_fwd on the mask the lists describe.
 *
 *  list      in   device int16 [B, H, T, T]: row (b, h, i) holds counts[b, h, i] key-tile indices,
 *                 strictly descending, each < T; bit 14 (0x4000) may tag an entry that must never
 *                 be flagged (a must-do tile). Entries past the count are not read.
 *  counts    in   device int32 [B, H, T], each in [0, T].
 *  mask_out  in/out device uint32 [B, H, T, W], or NULL = do not record flags. Flags are OR-ed into
 *                 it as they are found; nothing is copied into it first (initialise it, e.g. with
 *                 the mask the lists came from).
 *  Other arguments as lite_attn_fwd. Scratch (work order, counter: about 4*B*H*T bytes) comes from
 *  the library's stream-ordered pool, as for lite_attn_fwd.
 *
 * The attention kernel checks every list it walks: a count outside [0, T], an entry with bits other
 * than the index and the tag, an index >= T or one not below its predecessor stops the kernel
 * before that tile is loaded, and lite_get_device_status then returns LITE_ERR_CHECK (the outputs
 * of that call are invalid; the context stays usable).
 */
int lite_attn_fwd_list(const void* q, const void* k, const void* v, void* o, float* lse, const int16_t* list,
                       const int32_t* counts, uint32_t* mask_out, int B, int H, int N, int d, float scale, float tau,
                       lite_stream_t stream);

/*
 * lite_attn_fwd_ex -- lite_attn_fwd for partial attention: queries and keys of different lengths,
 * plus must-do / must-skip key-token ranges.
 *
 * Partial attention (README, LSE section): full self-attention over text and video tokens splits
 * into text-to-text, text-to-video, video-to-text and video-to-video pieces whose outputs combine
 * exactly by their LSE (lite_lse_merge). Each piece is this call with its own queries (Nq rows) and
 * keys / values (Nk rows); the skip test runs only where mask_out is given and tau > -inf (README:
 * skipping on for video-to-video, off for the others).
 *
 * Ranges (README, must_do_list / must_skip_list): a list [start_0, end_0, start_1, end_1, ...] of
 * key-token indices with start_0 > end_0 > start_1 > end_1 > ... (strictly descending, because
 * the key tiles are visited in reverse order) names the tokens end_i + 1 .. start_i of each pair
 * (start inclusive, end exclusive). Tokens at or beyond Nk are ignored.
 *   - A key tile holding at least one must-do token is live for every query tile whatever the
 *     mask says, and is never flagged (its mask_out bit is mask_in's).
 *   - A key tile whose tokens all lie inside must-skip ranges is skipped for every query tile (it
 *     is not added to mask_out either: the ranges are re-applied on every call).
 *   - Where both apply, must-do wins.
 *
 *  q          in   device bf16 [B, Nq, H, d].
 *  k, v       in   device bf16 [B, Nk, H, d].
 *  o          out  device bf16 [B, Nq, H, d].
 *  lse        out  device fp32 [B, H, Nq], or NULL.
 *  mask_in    in   device uint32 [B, H, Tq, Wk], or NULL = nothing skipped. Tq = ceil(Nq / tile),
 *                  Tk = ceil(Nk / tile), Wk = ceil(Tk / 32); bit j of a row = skip key tile j.
 *  mask_out   out  device uint32 [B, H, Tq, Wk], or NULL; may equal mask_in.
 *  must_do    in   HOST int32 array of n_must_do entries (even, >= 0), or NULL when n_must_do = 0.
 *  must_skip  in   HOST int32 array of n_must_skip entries, same convention.
 *                  The lists are read during the call only. A list that is not strictly
 *                  descending, has an odd length, or has an end below -1 is LITE_ERR_INVALID_ARG.
 *  B, H, Nq, Nk, d  Tq, Tk <= 4096; B*H <= 8192; d in {64, 128}.
 *  scale, tau, stream  as in lite_attn_fwd.
 * Scratch as in lite_attn_fwd (Tk entries per query tile in the live lists). lite_attn_fwd is this
 * call with Nq = Nk = N and no ranges.
 */
int lite_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse,
                     const uint32_t* mask_in, uint32_t* mask_out, const int32_t* must_do,
                     int n_must_do, const int32_t* must_skip, int n_must_skip, int B, int H, int Nq,
                     int Nk, int d, float scale, float tau, lite_stream_t stream);

/*
 * lite_attn_dense_ex -- lite_attn_dense with Nq query rows and Nk key rows (layouts as in
 * lite_attn_fwd_ex): the no-skip pieces of a partial attention. No mask, no scratch.
 */
int lite_attn_dense_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                       int H, int Nq, int Nk, int d, float scale, lite_stream_t stream);

/*
 * lite_lse_merge -- combine partial attentions over disjoint key sets (README, LSE section: the
 * partial results are combined with their LSE values).
 *
 * For every (b, h) and query row n, with parts p = 0 .. n_parts-1:
 *   lse = ln sum_p exp(lse_p),   o = sum_p exp(lse_p - lse) * o_p,
 * computed in fp32 from the bf16 partial outputs. Parts with lse_p = -inf for a row contribute
 * nothing; a row that is -inf in every part gets o = 0 and lse = -inf.
 *
 *  outs     in   HOST array of n_parts device pointers, each bf16 [B, N, H, d], 16-byte aligned.
 *  lses     in   HOST array of n_parts device pointers, each fp32 [B, H, N] (none NULL).
 *  n_parts       1 .. 8.
 *  o        out  device bf16 [B, N, H, d]; may be one of outs (in place).
 *  lse      out  device fp32 [B, H, N], or NULL; may be one of lses.
 *  B, H, N, d    d in {64, 128}; B*H*N*d/8 < 2^31 (LITE_ERR_UNSUPPORTED otherwise).
 * The two host arrays are read during the call only.
 */
int lite_lse_merge(const void* const* outs, const float* const* lses, int n_parts, void* o,
                   float* lse, int B, int H, int N, int d, lite_stream_t stream);

/*
 * lite_dropped_mass -- the error a Skip-Mask introduces at one step, for the accumulated-error
 * calibration of the QK-Skip threshold ("Lite Attention Temporal Sparse" skill page, Architecture
 * Overview: Accumulated-Error Calibration; README contribution list, "Error Calibration").
 *
 * For every (b, h) and query row n, the softmax probability that the skipped key tiles hold under
 * the dense softmax: 1 - exp(lse_live - lse_full), computed as -expm1 in fp32 and clamped to [0, 1];
 * a row whose lse_live is -inf (no live tile) drops 1.
 *
 *  lse_live  in   device fp32 [B, H, N]: lse of lite_attn_fwd with the mask as mask_in (tau = -inf).
 *  lse_full  in   device fp32 [B, H, N]: lse of lite_attn_dense on the same q, k, v.
 *  row_mass  out  device fp32 [B, H, N], or NULL.
 *  stats     out  device fp32 [2]: {largest per-row value, sum over all rows}. The call zeroes it
 *                 on `stream` first; read it after the stream has reached this call.
 *  Pointers must be 4-byte aligned (16-byte alignment of all three arrays enables vector loads).
 */
int lite_dropped_mass(const float* lse_live, const float* lse_full, float* row_mass, float* stats,
                      int B, int H, int N, lite_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* LITE_ATTN_H */
