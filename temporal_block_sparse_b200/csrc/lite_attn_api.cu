// lite_attn_api.cu -- host side of the C ABI declared in include/lite_attn.h.
//
// Validates arguments (before any CUDA call), builds the TMA tensor maps, takes stream-ordered
// scratch memory and enqueues: compaction (Skip-Mask -> Skip-List, mask copy, must-do / must-skip
// ranges) -> schedule (LPT work order) -> persistent attention. Also the LSE merge of partial
// attentions. Status words, options and per-device caches live here.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "attn_kernel.cuh"
#include "calib_kernels.cuh"
#include "lite_attn.h"
#include "mask_kernels.cuh"
#include "merge_kernel.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxT = 4096;

__device__ int g_device_status;  // one per device; set by kernels, read/cleared by the host

struct Options {
  unsigned long long wait_limit_ns = 4000000000ull;
  int debug_stall = 0;
  int max_ctas = 0;
  int schedule = 1;
  int pair_stride = 0;  // 0: chosen per call from the mask; k >= 1: query tiles r and r + k paired
};
Options g_opt;
unsigned long long* g_cta_times = nullptr;
int g_cta_cap = 0;
cudaEvent_t g_ev_before = nullptr;
cudaEvent_t g_ev_after = nullptr;
#ifdef LITE_ATTN_TRACE
long long* g_trace = nullptr;
#endif

struct DeviceCache {
  bool init = false;
  int dev = 0;
  int sms = 0;
  int* status = nullptr;
  bool smem_set[4] = {false, false, false, false};
  // Library-owned stream-ordered pool for per-call scratch. It keeps freed memory (release
  // threshold = max), so steady-state calls reuse it instead of mapping new memory, and it does
  // not alter the application's default pool.
  cudaMemPool_t pool = nullptr;
};
DeviceCache g_dev[kMaxDevices];
std::mutex g_mu;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

cudaStream_t as_stream(lite_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

// Per-device set-up that every entry point needs: SM count, the status word's device address and
// the tensor-map encoder. It allocates nothing; the scratch pool is created separately, on the first
// pooled call (ensure_pool).
int device_cache(DeviceCache** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LITE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceCache& c = g_dev[dev];
  if (!c.init) {
    if (cudaDeviceGetAttribute(&c.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return LITE_ERR_CUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void**>(&c.status), g_device_status) != cudaSuccess)
      return LITE_ERR_CUDA;
    c.dev = dev;
    c.init = true;
  }
  if (!g_encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return LITE_ERR_CUDA;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  *out = &c;
  return LITE_OK;
}

// The library-owned stream-ordered pool of a device, created on first use by a pooled call.
int ensure_pool(DeviceCache* c) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (c->pool) return LITE_OK;
  cudaMemPoolProps props;
  std::memset(&props, 0, sizeof(props));
  props.allocType = cudaMemAllocationTypePinned;
  props.location.type = cudaMemLocationTypeDevice;
  props.location.id = c->dev;
  cudaMemPool_t pool = nullptr;
  if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return LITE_ERR_CUDA;
  uint64_t keep = ~uint64_t(0);
  if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep) != cudaSuccess) {
    cudaMemPoolDestroy(pool);
    return LITE_ERR_CUDA;
  }
  c->pool = pool;
  return LITE_OK;
}

bool debug_env() {
  const char* e = std::getenv("LITE_ATTN_DEBUG");
  return e && std::strcmp(e, "FALSE") != 0;
}

int tile_for(int d) { return d == 64 ? 64 : (d == 128 ? 128 : 0); }

// Skip-Mask rows stacked in one 128-row kernel query tile: 2 for the 64-row tiles of d = 64.
int mask_rows_per_tile(int d) { return 128 / tile_for(d); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shapes(int B, int H, int Nq, int Nk, int d) {
  if (B <= 0 || H <= 0 || Nq <= 0 || Nk <= 0) return LITE_ERR_INVALID_ARG;
  const int t = tile_for(d);
  if (!t) return LITE_ERR_UNSUPPORTED;
  const long long Tq = (static_cast<long long>(Nq) + t - 1) / t;
  const long long Tk = (static_cast<long long>(Nk) + t - 1) / t;
  if (Tq > kMaxT || Tk > kMaxT) return LITE_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * Tq > (1ll << 30)) return LITE_ERR_UNSUPPORTED;
  return LITE_OK;
}

int check_shapes(int B, int H, int N, int d) { return check_shapes(B, H, N, N, d); }

int check_qkvo(const void* q, const void* k, const void* v, const void* o, const float* lse) {
  if (!q || !k || !v || !o) return LITE_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LITE_ERR_UNSUPPORTED;
  if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return LITE_ERR_UNSUPPORTED;
  return LITE_OK;
}

// [B, N, H, d] bf16 viewed as a 5-D tensor (64, N, d/64, H, B): the head dim is split into 64-element
// (128-byte) chunks and the chunk index is placed OUTSIDE the token index, so that one box of
// 64 x rows x d/64 lands in shared memory as d/64 consecutive [rows][128 B] swizzle-128B panels --
// the K-major operand layout of the MMA -- in a single TMA request per tile.
bool make_tmap(CUtensorMap* map, const void* ptr, int B, int N, int H, int d, int rows) {
  cuuint64_t dims[5] = {64, cuuint64_t(N), cuuint64_t(d / 64), cuuint64_t(H), cuuint64_t(B)};
  cuuint64_t strides[4] = {cuuint64_t(H) * d * 2, 128, cuuint64_t(d) * 2, cuuint64_t(N) * H * d * 2};
  cuuint32_t box[5] = {64, cuuint32_t(rows), cuuint32_t(d / 64), 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

float resolve_scale(float scale, int d) {
  if (!(scale > 0.f) || std::isnan(scale)) return 1.0f / std::sqrt(static_cast<float>(d));
  return scale;
}

template <int D, int BN>
int launch_attention(DeviceCache* dc, int cfg_slot, const void* q, const void* k, const void* v,
                     lite::AttnParams p, cudaStream_t stream) {
  using C = lite::AttnCfg<D, BN>;
  if (!dc->smem_set[cfg_slot]) {
    if (cudaFuncSetAttribute(lite::lite_attn_kernel<D, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::SMEM_BYTES) != cudaSuccess)
      return LITE_ERR_CUDA;
    dc->smem_set[cfg_slot] = true;
  }
  CUtensorMap tq, tk, tv, to;
  if (!make_tmap(&tq, q, p.B, p.Nq, p.H, D, C::BQ) || !make_tmap(&tk, k, p.B, p.Nk, p.H, D, BN) ||
      !make_tmap(&tv, v, p.B, p.Nk, p.H, D, BN) || !make_tmap(&to, p.o, p.B, p.Nq, p.H, D, C::OST_ROWS))
    return LITE_ERR_CUDA;
  int grid = dc->sms * C::CTAS_PER_SM;  // persistent: every resident CTA slot
  if (g_opt.max_ctas > 0 && g_opt.max_ctas < grid) grid = g_opt.max_ctas;
  if (p.n_items < grid) grid = p.n_items;
  if (grid <= 0) return LITE_OK;
  if (g_ev_before) cudaEventRecord(g_ev_before, stream);
  lite::lite_attn_kernel<D, BN><<<grid, C::THREADS, C::SMEM_BYTES, stream>>>(tq, tk, tv, to, p);
  if (cudaGetLastError() != cudaSuccess) return LITE_ERR_CUDA;
  if (g_ev_after) cudaEventRecord(g_ev_after, stream);
  return LITE_OK;
}

int run_attention(DeviceCache* dc, int d, const void* q, const void* k, const void* v, const lite::AttnParams& p,
                  cudaStream_t stream) {
  if (d == 64) return launch_attention<64, 64>(dc, 0, q, k, v, p, stream);
  return launch_attention<128, 128>(dc, 1, q, k, v, p, stream);
}

lite::AttnParams base_params(void* o, float* lse, int B, int H, int Nq, int Nk, int d, float scale,
                             DeviceCache* dc) {
  lite::AttnParams p;
  std::memset(&p, 0, sizeof(p));
  const int t = tile_for(d);
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.B = B;
  p.H = H;
  p.Nq = Nq;
  p.Nk = Nk;
  p.Tq = (Nq + t - 1) / t;
  p.Tk = (Nk + t - 1) / t;
  p.W = (p.Tk + 31) / 32;
  p.Tkq = (p.Tq + mask_rows_per_tile(d) - 1) / mask_rows_per_tile(d);  // kernel query tiles of 128 rows
  p.Pq = (p.Tkq + 1) / 2;
  p.n_items = B * H * p.Pq;  // work items: pairs of kernel query tiles
  p.pair_stride = 1;
  p.scale_log2 = resolve_scale(scale, d) * 1.4426950408889634f;
  p.tau_log2 = -INFINITY;
  p.status = dc->status;
  p.wait_limit_ns = g_opt.wait_limit_ns;
  p.debug_stall = g_opt.debug_stall;
  p.cta_times = g_cta_times;
  p.cta_cap = g_cta_cap;
#ifdef LITE_ATTN_TRACE
  p.trace = g_trace;
#endif
  return p;
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---- the masked forward pass, shared by lite_attn_fwd, lite_attn_fwd_ex and lite_attn_fwd_noalloc

struct FwdArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const uint32_t* mask_in;
  uint32_t* mask_out;
  int B, H, Nq, Nk, d;
  float scale, tau;
};

// every argument check that needs no CUDA call
int validate_fwd(const FwdArgs& a) {
  int st = check_qkvo(a.q, a.k, a.v, a.o, a.lse);
  if (st) return st;
  st = check_shapes(a.B, a.H, a.Nq, a.Nk, a.d);
  if (st) return st;
  if (std::isnan(a.tau)) return LITE_ERR_INVALID_ARG;
  if (a.tau > 0.f && !debug_env()) return LITE_ERR_INVALID_ARG;
  if ((a.mask_in && (reinterpret_cast<uintptr_t>(a.mask_in) & 3u)) ||
      (a.mask_out && (reinterpret_cast<uintptr_t>(a.mask_out) & 3u)))
    return LITE_ERR_UNSUPPORTED;
  if (static_cast<long long>(a.B) * a.H > 8192) return LITE_ERR_UNSUPPORTED;
  return LITE_OK;
}

// Scratch layout: live lists [rows, Tk] int16 | counts [rows] | order [rows] | a 512-byte tail with
// the work counter (+0), the chosen pairing stride (+4) and the stride scores (+256, 64 x uint32).
constexpr size_t kTailBytes = 512;
struct FwdScratch {
  size_t list_b, cnt_b, total;
};
struct Tail {
  int32_t* counter;
  int32_t* stride;
  uint32_t* scores;
};
Tail tail_at(char* t) {
  return Tail{reinterpret_cast<int32_t*>(t), reinterpret_cast<int32_t*>(t + 4), reinterpret_cast<uint32_t*>(t + 256)};
}

// Enqueues the pairing-stride choice (when the option leaves it to the mask) and the pair schedule;
// fills the attention parameters' work order, counter and stride.
int enqueue_pairs(const FwdArgs& a, const uint32_t* mask_in, const int32_t* counts, int32_t* order, char* tail,
                  lite::AttnParams& p, cudaStream_t s) {
  const Tail t = tail_at(tail);
  const int Tq = p.Tq, BH = a.B * a.H;
  const bool stacked = mask_rows_per_tile(a.d) == 2;
  // The stride is scored for one mask row per kernel query tile (d = 128); with stacked rows
  // (d = 64) the kernel query tiles are paired consecutively unless the option fixes a stride.
  const int n_cand = std::max(1, std::min(lite::kMaxPairStride, Tq / 2));
  const bool scored = !stacked && g_opt.pair_stride == 0 && mask_in != nullptr && n_cand > 1;
  if (scored) {
    const int chunks = std::max(1, std::min(8, BH));
    lite::lite_stride_score_kernel<<<dim3(n_cand, chunks), 256, 0, s>>>(mask_in, t.scores, BH, Tq, p.Tk, p.W);
    if (cudaGetLastError() != cudaSuccess) return LITE_ERR_CUDA;
  }
  if (g_opt.schedule) {
    const size_t sm = size_t(BH + p.Pq) * sizeof(int32_t);
    if (stacked)
      lite::lite_schedule_kernel<4><<<BH, 512, sm, s>>>(counts, order, BH, Tq, nullptr, 0, g_opt.pair_stride,
                                                        t.stride);
    else
      lite::lite_schedule_kernel<2><<<BH, 512, sm, s>>>(counts, order, BH, Tq, scored ? t.scores : nullptr, n_cand,
                                                        g_opt.pair_stride, t.stride);
    if (cudaGetLastError() != cudaSuccess) return LITE_ERR_CUDA;
    p.pair_stride_ptr = t.stride;  // written by the schedule kernel
  } else {
    p.pair_stride_ptr = nullptr;
    p.pair_stride = g_opt.pair_stride >= 1 ? g_opt.pair_stride : 1;
  }
  p.order = g_opt.schedule ? order : nullptr;  // null: pairs in their natural order
  p.work_counter = t.counter;
  return LITE_OK;
}

FwdScratch fwd_scratch(const FwdArgs& a) {
  const int t = tile_for(a.d);
  const size_t Tq = (a.Nq + t - 1) / t, Tk = (a.Nk + t - 1) / t;
  const size_t rows = size_t(a.B) * a.H * Tq;
  FwdScratch f;
  f.list_b = align256(rows * Tk * sizeof(int16_t));
  f.cnt_b = align256(rows * sizeof(int32_t));
  f.total = f.list_b + 2 * f.cnt_b + kTailBytes;
  return f;
}

// README-style range list -> key-tile bitmap. whole = false: tiles holding any listed token
// (must-do); whole = true: tiles all of whose tokens are listed (must-skip). The list must be
// strictly descending (start_0 > end_0 > start_1 > ...), of even length, with ends >= -1; the
// strict order leaves at least one unlisted token between two ranges, so a tile covered by the
// union of the ranges is covered by one of them.
int range_bits(const int32_t* r, int n, int Nk, int t, bool whole, uint32_t* bits) {
  if (n < 0 || (n & 1) || (n > 0 && !r)) return LITE_ERR_INVALID_ARG;
  for (int x = 1; x < n; ++x)
    if (!(r[x - 1] > r[x])) return LITE_ERR_INVALID_ARG;
  if (n > 0 && r[n - 1] < -1) return LITE_ERR_INVALID_ARG;
  for (int x = 0; x < n; x += 2) {
    const long long lo = std::max(static_cast<long long>(r[x + 1]) + 1, 0ll);
    const long long hi = std::min(static_cast<long long>(r[x]), static_cast<long long>(Nk) - 1);
    if (lo > hi) continue;
    for (long long j = lo / t; j <= hi / t; ++j) {
      if (whole) {
        const long long c0 = j * t, c1 = std::min((j + 1) * t, static_cast<long long>(Nk)) - 1;
        if (c0 < lo || c1 > hi) continue;
      }
      bits[j >> 5] |= 1u << (j & 31);
    }
  }
  return LITE_OK;
}

// Enqueues compaction, schedule and attention with the given scratch (fwd_scratch layout).
int enqueue_fwd(DeviceCache* dc, const FwdArgs& a, const lite::RangeBits* ranges, char* base, cudaStream_t s) {
  const FwdScratch f = fwd_scratch(a);
  lite::AttnParams p = base_params(a.o, a.lse, a.B, a.H, a.Nq, a.Nk, a.d, a.scale, dc);
  const int Tq = p.Tq, Tk = p.Tk, W = p.W, rows = a.B * a.H * Tq;
  int16_t* list = reinterpret_cast<int16_t*>(base);
  int32_t* counts = reinterpret_cast<int32_t*>(base + f.list_b);
  int32_t* order = reinterpret_cast<int32_t*>(base + f.list_b + f.cnt_b);
  char* tail = base + f.list_b + 2 * f.cnt_b;

  // the work counter and the stride scores must start at zero (fixed scratch keeps the last call's)
  if (cudaMemsetAsync(tail, 0, kTailBytes, s) != cudaSuccess) return LITE_ERR_CUDA;
  const int cblocks = (rows + 7) / 8;
  if (ranges)
    lite::lite_compact_kernel<true><<<cblocks, 256, 0, s>>>(a.mask_in, a.mask_out, list, counts, rows, Tk, W, *ranges);
  else
    lite::lite_compact_kernel<false><<<cblocks, 256, 0, s>>>(a.mask_in, a.mask_out, list, counts, rows, Tk, W,
                                                             lite::RangeBits{});
  if (cudaGetLastError() != cudaSuccess) return LITE_ERR_CUDA;
  int st = enqueue_pairs(a, a.mask_in, counts, order, tail, p, s);
  if (st) return st;
  p.mask_out = a.mask_out;
  p.list = list;
  p.counts = counts;
  p.tau_log2 = a.tau * 1.4426950408889634f;
  p.skip_test = (a.mask_out != nullptr && a.tau > -INFINITY) ? 1 : 0;
  return run_attention(dc, a.d, a.q, a.k, a.v, p, s);
}

// Schedule and attention over caller-supplied Skip-Lists (no compaction, no mask copy). Scratch:
// work order [rows] int32 | work counter.
size_t list_scratch_bytes(const FwdArgs& a) {
  const int t = tile_for(a.d);
  const size_t rows = size_t(a.B) * a.H * ((a.Nq + t - 1) / t);
  return align256(rows * sizeof(int32_t)) + kTailBytes;
}

int enqueue_list(DeviceCache* dc, const FwdArgs& a, const int16_t* list, const int32_t* counts, char* base,
                 cudaStream_t s) {
  lite::AttnParams p = base_params(a.o, a.lse, a.B, a.H, a.Nq, a.Nk, a.d, a.scale, dc);
  const int rows = a.B * a.H * p.Tq;
  int32_t* order = reinterpret_cast<int32_t*>(base);
  char* tail = base + align256(size_t(rows) * sizeof(int32_t));
  if (cudaMemsetAsync(tail, 0, kTailBytes, s) != cudaSuccess) return LITE_ERR_CUDA;
  // no mask here: the pairing stride is the option's, or 1
  int st = enqueue_pairs(a, nullptr, counts, order, tail, p, s);
  if (st) return st;
  p.mask_out = a.mask_out;
  p.list = list;
  p.counts = counts;
  p.tau_log2 = a.tau * 1.4426950408889634f;
  p.skip_test = (a.mask_out != nullptr && a.tau > -INFINITY) ? 1 : 0;
  return run_attention(dc, a.d, a.q, a.k, a.v, p, s);
}

// pool-backed scratch around enqueue_fwd
int fwd_pooled(const FwdArgs& a, const lite::RangeBits* ranges, cudaStream_t s) {
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK || ensure_pool(dc) != LITE_OK) return LITE_ERR_CUDA;
  const FwdScratch f = fwd_scratch(a);
  void* ws = nullptr;
  if (cudaMallocFromPoolAsync(&ws, f.total, dc->pool, s) != cudaSuccess) return LITE_ERR_CUDA;
  int st = enqueue_fwd(dc, a, ranges, static_cast<char*>(ws), s);
  if (cudaFreeAsync(ws, s) != cudaSuccess && !st) st = LITE_ERR_CUDA;
  return st;
}

}  // namespace

extern "C" {

int lite_mask_geometry(int N, int d, int* tile, int* T, int* words) {
  if (N <= 0) return LITE_ERR_INVALID_ARG;
  const int t = tile_for(d);
  if (!t) return LITE_ERR_UNSUPPORTED;
  const int TT = (N + t - 1) / t;
  if (tile) *tile = t;
  if (T) *T = TT;
  if (words) *words = (TT + 31) / 32;
  return LITE_OK;
}

const char* lite_status_string(int status) {
  switch (status) {
    case LITE_OK: return "ok";
    case LITE_ERR_INVALID_ARG: return "invalid argument";
    case LITE_ERR_UNSUPPORTED: return "unsupported shape, head dim or alignment";
    case LITE_ERR_CUDA: return "CUDA launch, allocation or query failed";
    case LITE_ERR_TIMEOUT: return "a kernel wait exceeded its time limit; outputs of that call are invalid";
    case LITE_ERR_CHECK: return "a kernel found a malformed Skip-List, live count or work order; outputs of that call are invalid";
    case LITE_ERR_SCRATCH_LIMIT: return "layer needs more scratch than lite_attn_fwd_noalloc's fixed 8 MiB";
    default: return "unknown status";
  }
}

int lite_set_option(int option, long long value) {
  switch (option) {
    case LITE_OPT_WAIT_LIMIT_NS:
      if (value < 1000) return LITE_ERR_INVALID_ARG;
      g_opt.wait_limit_ns = static_cast<unsigned long long>(value);
      return LITE_OK;
    case LITE_OPT_DEBUG_STALL:
      if (value != 0 && value != 1) return LITE_ERR_INVALID_ARG;
      g_opt.debug_stall = static_cast<int>(value);
      return LITE_OK;
    case LITE_OPT_SCHEDULE:
      if (value != 0 && value != 1) return LITE_ERR_INVALID_ARG;
      g_opt.schedule = int(value);
      return LITE_OK;
    case LITE_OPT_MAX_CTAS:
      if (value < 0 || value > 1000000) return LITE_ERR_INVALID_ARG;
      g_opt.max_ctas = static_cast<int>(value);
      return LITE_OK;
    case LITE_OPT_PAIR_STRIDE:
      if (value < 0 || value > kMaxT) return LITE_ERR_INVALID_ARG;
      g_opt.pair_stride = static_cast<int>(value);
      return LITE_OK;
    default:
      return LITE_ERR_INVALID_ARG;
  }
}

int lite_set_cta_timing(void* buf, int capacity) {
  if ((buf == nullptr) != (capacity == 0) || capacity < 0) return LITE_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(buf) & 7u) return LITE_ERR_UNSUPPORTED;
  g_cta_times = static_cast<unsigned long long*>(buf);
  g_cta_cap = capacity;
  return LITE_OK;
}

int lite_set_kernel_events(void* before, void* after) {
  if ((before == nullptr) != (after == nullptr)) return LITE_ERR_INVALID_ARG;
  g_ev_before = static_cast<cudaEvent_t>(before);
  g_ev_after = static_cast<cudaEvent_t>(after);
  return LITE_OK;
}

int lite_scratch_pool_bytes(long long* reserved) {
  if (!reserved) return LITE_ERR_INVALID_ARG;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  *reserved = 0;
  if (!dc->pool) return LITE_OK;
  cuuint64_t v = 0;
  if (cudaMemPoolGetAttribute(dc->pool, cudaMemPoolAttrReservedMemCurrent, &v) != cudaSuccess) return LITE_ERR_CUDA;
  *reserved = static_cast<long long>(v);
  return LITE_OK;
}

int lite_get_device_status(lite_stream_t stream) {
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return LITE_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, dc->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LITE_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(dc->status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return LITE_ERR_CUDA;
  }
  return v;
}

int lite_mask_to_list(const uint32_t* mask, int16_t* list, int32_t* counts, int B, int H, int N, int d,
                      lite_stream_t stream) {
  if (!list || !counts) return LITE_ERR_INVALID_ARG;
  int st = check_shapes(B, H, N, d);
  if (st) return st;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  const int t = tile_for(d), T = (N + t - 1) / t, W = (T + 31) / 32;
  const int rows = B * H * T;
  lite::lite_compact_kernel<false><<<(rows + 7) / 8, 256, 0, as_stream(stream)>>>(mask, nullptr, list, counts, rows,
                                                                                  T, W, lite::RangeBits{});
  return cudaGetLastError() == cudaSuccess ? LITE_OK : LITE_ERR_CUDA;
}

int lite_mask_to_ranges(const uint32_t* mask, int16_t* ranges, int32_t* nruns, int B, int H, int N, int d,
                        lite_stream_t stream) {
  if (!ranges || !nruns) return LITE_ERR_INVALID_ARG;
  int st = check_shapes(B, H, N, d);
  if (st) return st;
  if (reinterpret_cast<uintptr_t>(ranges) & 1u || reinterpret_cast<uintptr_t>(nruns) & 3u ||
      reinterpret_cast<uintptr_t>(mask) & 3u)
    return LITE_ERR_UNSUPPORTED;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  const int t = tile_for(d), T = (N + t - 1) / t, W = (T + 31) / 32;
  const int rows = B * H * T;
  lite::lite_ranges_kernel<<<(rows + 7) / 8, 256, 0, as_stream(stream)>>>(mask, ranges, nruns, rows, T, W);
  return cudaGetLastError() == cudaSuccess ? LITE_OK : LITE_ERR_CUDA;
}

int lite_schedule(const int32_t* counts, int32_t* order, int B, int H, int T, lite_stream_t stream) {
  if (!counts || !order || B <= 0 || H <= 0 || T <= 0) return LITE_ERR_INVALID_ARG;
  if (static_cast<long long>(B) * H > 8192 || T > kMaxT) return LITE_ERR_UNSUPPORTED;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  const int BH = B * H;
  const size_t sm = size_t(BH + T) * sizeof(int32_t);
  lite::lite_schedule_kernel<1><<<BH, 512, sm, as_stream(stream)>>>(counts, order, BH, T);
  return cudaGetLastError() == cudaSuccess ? LITE_OK : LITE_ERR_CUDA;
}

int lite_attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, const uint32_t* mask_in,
                  uint32_t* mask_out, int B, int H, int N, int d, float scale, float tau, lite_stream_t stream) {
  const FwdArgs a{q, k, v, o, lse, mask_in, mask_out, B, H, N, N, d, scale, tau};
  const int st = validate_fwd(a);
  if (st) return st;
  return fwd_pooled(a, nullptr, as_stream(stream));
}

int lite_attn_fwd_list(const void* q, const void* k, const void* v, void* o, float* lse, const int16_t* list,
                       const int32_t* counts, uint32_t* mask_out, int B, int H, int N, int d, float scale, float tau,
                       lite_stream_t stream) {
  const FwdArgs a{q, k, v, o, lse, nullptr, mask_out, B, H, N, N, d, scale, tau};
  int st = validate_fwd(a);
  if (st) return st;
  if (!list || !counts) return LITE_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(list) & 1u) || (reinterpret_cast<uintptr_t>(counts) & 3u))
    return LITE_ERR_UNSUPPORTED;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK || ensure_pool(dc) != LITE_OK) return LITE_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  void* ws = nullptr;
  if (cudaMallocFromPoolAsync(&ws, list_scratch_bytes(a), dc->pool, s) != cudaSuccess) return LITE_ERR_CUDA;
  st = enqueue_list(dc, a, list, counts, static_cast<char*>(ws), s);
  if (cudaFreeAsync(ws, s) != cudaSuccess && !st) st = LITE_ERR_CUDA;
  return st;
}

int lite_attn_fwd_ex(const void* q, const void* k, const void* v, void* o, float* lse, const uint32_t* mask_in,
                     uint32_t* mask_out, const int32_t* must_do, int n_must_do, const int32_t* must_skip,
                     int n_must_skip, int B, int H, int Nq, int Nk, int d, float scale, float tau,
                     lite_stream_t stream) {
  const FwdArgs a{q, k, v, o, lse, mask_in, mask_out, B, H, Nq, Nk, d, scale, tau};
  int st = validate_fwd(a);
  if (st) return st;
  lite::RangeBits rb;
  std::memset(&rb, 0, sizeof(rb));
  const int t = tile_for(d);
  st = range_bits(must_do, n_must_do, Nk, t, false, rb.live);
  if (st) return st;
  st = range_bits(must_skip, n_must_skip, Nk, t, true, rb.skip);
  if (st) return st;
  for (int w = 0; w < 128; ++w) rb.skip[w] &= ~rb.live[w];  // must-do wins
  const bool any = n_must_do > 0 || n_must_skip > 0;
  return fwd_pooled(a, any ? &rb : nullptr, as_stream(stream));
}

int lite_attn_dense_ex(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                       int Nk, int d, float scale, lite_stream_t stream) {
  int st = check_qkvo(q, k, v, o, lse);
  if (st) return st;
  st = check_shapes(B, H, Nq, Nk, d);
  if (st) return st;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  lite::AttnParams p = base_params(o, lse, B, H, Nq, Nk, d, scale, dc);
  // every tile live, identity order, static striding over items (uniform cost): no scratch
  return run_attention(dc, d, q, k, v, p, as_stream(stream));
}

int lite_attn_dense(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                    float scale, lite_stream_t stream) {
  return lite_attn_dense_ex(q, k, v, o, lse, B, H, N, N, d, scale, stream);
}

int lite_lse_merge(const void* const* outs, const float* const* lses, int n_parts, void* o, float* lse, int B,
                   int H, int N, int d, lite_stream_t stream) {
  if (!outs || !lses || !o || n_parts < 1 || B <= 0 || H <= 0 || N <= 0) return LITE_ERR_INVALID_ARG;
  if (n_parts > lite::kMaxMergeParts) return LITE_ERR_UNSUPPORTED;
  if (d != 64 && d != 128) return LITE_ERR_UNSUPPORTED;
  lite::MergeParts mp;
  std::memset(&mp, 0, sizeof(mp));
  for (int x = 0; x < n_parts; ++x) {
    if (!outs[x] || !lses[x]) return LITE_ERR_INVALID_ARG;
    if (!aligned16(outs[x]) || (reinterpret_cast<uintptr_t>(lses[x]) & 3u)) return LITE_ERR_UNSUPPORTED;
    mp.o[x] = static_cast<const __nv_bfloat16*>(outs[x]);
    mp.lse[x] = lses[x];
  }
  mp.n = n_parts;
  if (!aligned16(o) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u))) return LITE_ERR_UNSUPPORTED;
  if (static_cast<long long>(B) * H * N * (d / 8) >= (1ll << 31)) return LITE_ERR_UNSUPPORTED;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  const long long threads = static_cast<long long>(B) * H * N * (d / 8);
  const long long want = (threads + 255) / 256;
  // grid-stride; up to 8 resident 256-thread blocks per SM
  const int blocks = int(std::min<long long>(want, static_cast<long long>(dc->sms) * 8));
  cudaStream_t s = as_stream(stream);
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(o);
  if (d == 64) {
    if (n_parts <= 2) lite::lite_lse_merge_kernel<64, 2><<<blocks, 256, 0, s>>>(mp, ob, lse, B, H, N);
    else if (n_parts <= 4) lite::lite_lse_merge_kernel<64, 4><<<blocks, 256, 0, s>>>(mp, ob, lse, B, H, N);
    else lite::lite_lse_merge_kernel<64, 8><<<blocks, 256, 0, s>>>(mp, ob, lse, B, H, N);
  } else {
    if (n_parts <= 2) lite::lite_lse_merge_kernel<128, 2><<<blocks, 256, 0, s>>>(mp, ob, lse, B, H, N);
    else if (n_parts <= 4) lite::lite_lse_merge_kernel<128, 4><<<blocks, 256, 0, s>>>(mp, ob, lse, B, H, N);
    else lite::lite_lse_merge_kernel<128, 8><<<blocks, 256, 0, s>>>(mp, ob, lse, B, H, N);
  }
  return cudaGetLastError() == cudaSuccess ? LITE_OK : LITE_ERR_CUDA;
}

int lite_dropped_mass(const float* lse_live, const float* lse_full, float* row_mass, float* stats, int B, int H,
                      int N, lite_stream_t stream) {
  if (!lse_live || !lse_full || !stats || B <= 0 || H <= 0 || N <= 0) return LITE_ERR_INVALID_ARG;
  const uintptr_t mis = reinterpret_cast<uintptr_t>(lse_live) | reinterpret_cast<uintptr_t>(lse_full) |
                        reinterpret_cast<uintptr_t>(row_mass) | reinterpret_cast<uintptr_t>(stats);
  if (mis & 3u) return LITE_ERR_UNSUPPORTED;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  cudaStream_t s = as_stream(stream);
  const long long rows = static_cast<long long>(B) * H * N;
  if (cudaMemsetAsync(stats, 0, 2 * sizeof(float), s) != cudaSuccess) return LITE_ERR_CUDA;
  const long long want = (rows + 1023) / 1024;  // 4 rows per thread, 256 threads per block
  const int blocks = int(std::max<long long>(1, std::min<long long>(want, static_cast<long long>(dc->sms) * 8)));
  lite::lite_dropped_mass_kernel<<<blocks, 256, 0, s>>>(lse_live, lse_full, row_mass, stats, rows);
  return cudaGetLastError() == cudaSuccess ? LITE_OK : LITE_ERR_CUDA;
}

#ifdef LITE_ATTN_TRACE
// analysis builds only: clock64 probes of the first CTAs go to this device buffer
int lite_trace_set(void* buf) {
  g_trace = static_cast<long long*>(buf);
  return LITE_OK;
}
#endif

}  // extern "C"

// ------------------------------------------------------------------------------------------------
// No-allocation variant of lite_attn_fwd.
//
// Its scratch lives in the file-scope device array below, which every device holds once the
// library is loaded on it. In host code `g_noalloc_scratch` is only a host-side stand-in for the
// symbol, not a device address: its device address is looked up once per device with
// cudaGetSymbolAddress (device current) and that address is what the kernels receive.

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[LITE_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_addr[kMaxDevices] = {nullptr};

// First call on a device: find the array's device address. Returns nullptr on failure.
void* noalloc_scratch() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_noalloc_addr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return nullptr;
    g_noalloc_addr[dev] = ptr;
  }
  return g_noalloc_addr[dev];
}

}  // namespace

extern "C" int lite_attn_fwd_noalloc(const void* q, const void* k, const void* v, void* o, float* lse,
                                     const uint32_t* mask_in, uint32_t* mask_out, int B, int H, int N, int d,
                                     float scale, float tau, lite_stream_t stream) {
  const FwdArgs a{q, k, v, o, lse, mask_in, mask_out, B, H, N, N, d, scale, tau};
  const int st = validate_fwd(a);
  if (st) return st;
  if (fwd_scratch(a).total > LITE_NOALLOC_SCRATCH_BYTES) return LITE_ERR_SCRATCH_LIMIT;
  DeviceCache* dc = nullptr;
  if (device_cache(&dc) != LITE_OK) return LITE_ERR_CUDA;
  char* base = static_cast<char*>(noalloc_scratch());
  if (!base) return LITE_ERR_CUDA;
  return enqueue_fwd(dc, a, nullptr, base, as_stream(stream));
}
