// C ABI of the MoGA layer library (declarations and contracts in moga.h).
// Host side only: argument validation, workspace carving, TMA descriptor
// encoding and kernel sequencing.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <mutex>

#include "../../include/moga.h"
#include "internal.h"

namespace moga {

namespace {

std::atomic<uint64_t> g_wait_ns{4000000000ull};
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_debug_inject{0};
constexpr int kNumStages = 6;
std::atomic<void*> g_ev_begin[kNumStages];
std::atomic<void*> g_ev_end[kNumStages];

// Records the optional timing event of `stage` on the call's stream.
void mark(int stage, bool begin, cudaStream_t s) {
  void* ev = (begin ? g_ev_begin : g_ev_end)[stage].load(std::memory_order_relaxed);
  if (ev) cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev), s);
}
void count(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms_of(int dev) {
  static std::atomic<int> cache[64];
  if (dev < 0 || dev >= 64) return 148;
  int v = cache[dev].load(std::memory_order_relaxed);
  if (v > 0) return v;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
  cache[dev].store(v, std::memory_order_relaxed);
  return v;
}

// ------------------------------------------------------------------ allocation-free routing scratch
// Scratch of moga_route_noalloc: the routing tile histograms and bases live in
// this file-scope device array instead of a caller workspace.  Every GPU that
// loads the library holds it (about 2 MiB) until the process exits.  Host code
// must not pass the symbol itself to a kernel (on the host it only names a
// stand-in); its device address comes from cudaGetSymbolAddress below.
constexpr int64_t kNoAllocCells = (int64_t)1 << 18;  // max ceil(N/128) * M
constexpr size_t kNoAllocBytes = 256 + 2 * (size_t)kNoAllocCells * 4;
static __device__ __align__(256) uint8_t g_route_scratch[kNoAllocBytes];

// The driver's cuCtxGetCurrent, resolved at run time like the tensor-map encoder.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(p);
  });
  return fn;
}

// Device address of g_route_scratch for the current device, looked up once per
// device and context (the first call on a device does it; see moga.h).  The
// context is part of the key: after a device reset the runtime loads the
// module again in a new context, where the array may sit elsewhere.
uint8_t* noalloc_scratch(int dev) {
  static std::mutex mu;
  static uint8_t* addr[64] = {};
  static CUcontext ctx_of[64] = {};
  if (dev < 0 || dev >= 64) return nullptr;
  const CtxGetCurrentFn get = ctx_get_current();
  if (!get) return nullptr;
  // null while this thread has no current context yet; the lookup below then
  // makes the device's primary context current
  CUcontext ctx = nullptr;
  if (get(&ctx) != CUDA_SUCCESS) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev] || !ctx || ctx_of[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return nullptr;
    if (get(&ctx) != CUDA_SUCCESS) return nullptr;
    addr[dev] = static_cast<uint8_t*>(p);
    ctx_of[dev] = ctx;
  }
  return addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

constexpr size_t kHeader = 256;  // status word and spare words

// Sequential 256-byte aligned carving of a workspace after its header.
struct Carve {
  size_t off = kHeader;
  size_t take(size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  }
};

struct RouteWs {
  size_t hist, base, pstat, total;
};
// with_stats adds the per-(tile, warp) sums of routing probabilities.
RouteWs route_ws(int64_t N, int M, bool with_stats = false) {
  Carve c;
  RouteWs w;
  const size_t cells = (size_t)ceil_div(N, kTile) * (size_t)M;
  w.hist = c.take(cells * 4);
  w.base = c.take(cells * 4);
  w.pstat = with_stats ? c.take(cells * 4 * 4) : 0;
  w.total = c.off;
  return w;
}

// Grouped attention (and windows larger than two query tiles) streams each
// segment's K/V many times, so it reads a gathered head-major copy of Q/K/V
// with tiled loads; small STGA windows read q, k, v in place by token index.
constexpr int64_t kDirectWindowMax = 2 * kTile;

struct AttnWs {
  size_t table, permw, qh, kh, vh, total;
};
AttnWs attn_ws(int64_t N, int H, int d_h, int nseg_table, bool window_perm, bool copy = true) {
  Carve c;
  AttnWs w;
  w.table = c.take((size_t)(3 * nseg_table + 1) * 4);
  w.permw = window_perm ? c.take((size_t)N * 4) : 0;
  w.qh = w.kh = w.vh = 0;
  if (copy) {
    const size_t mat = (size_t)N * H * d_h * 2;
    w.qh = c.take(mat);
    w.kh = c.take(mat);
    w.vh = c.take(mat);
  }
  w.total = c.off;
  return w;
}

bool stga_direct(const int* window) { return (int64_t)window[0] * window[1] * window[2] <= kDirectWindowMax; }

moga_status from_cuda(cudaError_t e) { return e == cudaSuccess ? MOGA_OK : MOGA_ERR_CUDA; }

bool make_ctx(DevCtx* c, void* ws, void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  c->device = dev;
  c->num_sms = num_sms_of(dev);
  c->stream = reinterpret_cast<cudaStream_t>(stream);
  c->status = reinterpret_cast<int*>(ws);
  c->wait_ns = g_wait_ns.load(std::memory_order_relaxed);
  return true;
}

moga_status check_attn_shape(int64_t N, int H, int d_h) {
  if (N < 0 || H < 1) return MOGA_ERR_INVALID_ARG;
  if (d_h != 64 && d_h != 128) return MOGA_ERR_UNSUPPORTED;
  if (N * (int64_t)H >= (int64_t)1 << 31) return MOGA_ERR_UNSUPPORTED;
  return MOGA_OK;
}

moga_status check_window(int T, int Hg, int Wg, const int* window, int64_t* N) {
  if (!window || T < 1 || Hg < 1 || Wg < 1) return MOGA_ERR_INVALID_ARG;
  if (window[0] < 1 || window[1] < 1 || window[2] < 1) return MOGA_ERR_INVALID_ARG;
  const int64_t n = (int64_t)T * Hg * Wg;
  if (n >= (int64_t)1 << 31) return MOGA_ERR_UNSUPPORTED;
  *N = n;
  return MOGA_OK;
}

// ------------------------------------------------------------------ bodies (args already validated)
moga_status route_body(const DevCtx& c, const void* x, const void* W, const float* b, moga_dtype dt, int64_t N,
                       int d, int M, int32_t* gid, float* gate, int32_t* perm, int32_t* offsets,
                       int32_t* max_seqlen, uint8_t* ws, float* prob_mean = nullptr, float* balance = nullptr) {
  const bool stats = prob_mean || balance;
  if (N == 0) {
    cudaError_t e = cudaMemsetAsync(offsets, 0, (size_t)(M + 1) * 4, c.stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(max_seqlen, 0, 4, c.stream);
    if (e == cudaSuccess && prob_mean) e = cudaMemsetAsync(prob_mean, 0, (size_t)M * 4, c.stream);
    if (e == cudaSuccess && balance) e = cudaMemsetAsync(balance, 0, 4, c.stream);
    return from_cuda(e);
  }
  const RouteWs w = route_ws(N, M, stats);
  int32_t* hist = reinterpret_cast<int32_t*>(ws + w.hist);
  int32_t* base = reinterpret_cast<int32_t*>(ws + w.base);
  float* pstat = stats ? reinterpret_cast<float*>(ws + w.pstat) : nullptr;
  cudaError_t e;
  mark(MOGA_STAGE_ROUTER, true, c.stream);
  if (dt == MOGA_BF16 && M <= 256 && d >= 64)
    e = launch_route_tc(c, x, W, b, N, d, M, gid, gate, hist, pstat);
  else
    e = launch_route_simt(c, x, W, b, dt == MOGA_BF16, N, d, M, gid, gate, hist, pstat);
  mark(MOGA_STAGE_ROUTER, false, c.stream);
  if (e != cudaSuccess) return MOGA_ERR_CUDA;
  mark(MOGA_STAGE_SORT, true, c.stream);
  if ((e = launch_scan(c, hist, ceil_div(N, kTile), M, base, offsets, max_seqlen, pstat, N, prob_mean,
                       balance)) != cudaSuccess)
    return MOGA_ERR_CUDA;
  if ((e = launch_scatter(c, gid, base, N, M, perm)) != cudaSuccess) return MOGA_ERR_CUDA;
  mark(MOGA_STAGE_SORT, false, c.stream);
  count(3);
  return MOGA_OK;
}

moga_status group_attn_body(const DevCtx& c, const void* q, const void* k, const void* v, const int32_t* perm,
                            const int32_t* offsets, const float* gate, int64_t N, int H, int d_h, int M,
                            float out_scale, void* out, uint8_t* ws, float* lse = nullptr) {
  if (N == 0) return MOGA_OK;
  const AttnWs w = attn_ws(N, H, d_h, M, false);
  int32_t* table = reinterpret_cast<int32_t*>(ws + w.table);
  mark(MOGA_STAGE_GATHER, true, c.stream);
  if (launch_seg_table(c, offsets, M, H, N, table) != cudaSuccess) return MOGA_ERR_CUDA;
  if (launch_gather(c, q, k, v, perm, N, H, d_h, ws + w.qh, ws + w.kh, ws + w.vh) != cudaSuccess)
    return MOGA_ERR_CUDA;
  mark(MOGA_STAGE_GATHER, false, c.stream);
  count(2);
  AttnArgs a{};
  a.direct = 0;
  a.q = ws + w.qh;
  a.k = ws + w.kh;
  a.v = ws + w.vh;
  a.perm = perm;
  a.gate = gate;
  a.out = out;
  a.N = N;
  a.H = H;
  a.d_h = d_h;
  a.out_scale = out_scale;
  a.accumulate = 0;
  a.mode = 0;
  a.table = table;
  a.nseg = M;
  a.lse = lse;
  a.debug_withhold_first_k = g_debug_inject.load(std::memory_order_relaxed) == 1;
  mark(MOGA_STAGE_GROUP_ATTN, true, c.stream);
  const cudaError_t e = launch_attention(c, a);
  mark(MOGA_STAGE_GROUP_ATTN, false, c.stream);
  count(1);
  return from_cuda(e);
}

// accumulate == 0: out = STGA; otherwise out += add_scale * STGA.
moga_status stga_body(const DevCtx& c, const void* q, const void* k, const void* v, int T, int Hg, int Wg,
                      const int* window, int H, int d_h, int accumulate, void* out, uint8_t* ws,
                      float add_scale = 0.5f, float* lse = nullptr) {
  const int64_t N = (int64_t)T * Hg * Wg;
  const bool direct = stga_direct(window);
  // Windows of whole frames are runs of consecutive tokens: no permutation,
  // no gathered copy, the tiled kernel reads q, k, v in place.
  const bool contiguous = !direct && window[1] >= Hg && window[2] >= Wg;
  const AttnWs w = attn_ws(N, H, d_h, 0, true, !direct);
  int32_t* permw = reinterpret_cast<int32_t*>(ws + w.permw);
  // Small windows are loaded as whole TMA boxes (stga.cu) and need no
  // permutation, except for the training forward, whose log-sum-exp rows
  // (and the backward pass after it) follow the window order.
  const bool box = stga_box_supported(d_h, window);
  mark(MOGA_STAGE_STGA_PREP, true, c.stream);
  if (!contiguous && (!box || lse)) {
    if (launch_window_perm(c, T, Hg, Wg, window, permw) != cudaSuccess) return MOGA_ERR_CUDA;
    count(1);
  }
  AttnArgs a{};
  a.direct = direct ? 1 : 0;
  a.contiguous = contiguous ? 1 : 0;
  if (direct || contiguous) {
    a.q = q;
    a.k = k;
    a.v = v;
  } else {
    if (launch_gather(c, q, k, v, permw, N, H, d_h, ws + w.qh, ws + w.kh, ws + w.vh) != cudaSuccess)
      return MOGA_ERR_CUDA;
    count(1);
    a.q = ws + w.qh;
    a.k = ws + w.kh;
    a.v = ws + w.vh;
  }
  mark(MOGA_STAGE_STGA_PREP, false, c.stream);
  a.perm = contiguous ? nullptr : permw;
  a.gate = nullptr;
  a.out = out;
  a.N = N;
  a.H = H;
  a.d_h = d_h;
  a.out_scale = accumulate ? add_scale : 1.0f;
  a.accumulate = accumulate ? 1 : 0;
  a.mode = 1;
  a.table = nullptr;
  a.nseg = (int)stga_num_windows(T, Hg, Wg, window);
  a.T = T;
  a.Hg = Hg;
  a.Wg = Wg;
  a.wt = window[0];
  a.wh = window[1];
  a.ww = window[2];
  a.lse = lse;
  a.debug_withhold_first_k = g_debug_inject.load(std::memory_order_relaxed) == 1;
  mark(MOGA_STAGE_STGA_ATTN, true, c.stream);
  bool handled = false;
  cudaError_t e = box ? launch_stga_box(c, a, &handled) : cudaSuccess;
  if (e == cudaSuccess && !handled) {
    if (box && !lse && !contiguous) {
      // the box kernel declined (tensor map not encodable): the general
      // kernel reads rows by the window permutation
      if (launch_window_perm(c, T, Hg, Wg, window, permw) != cudaSuccess) return MOGA_ERR_CUDA;
      count(1);
    }
    e = launch_attention(c, a);
  }
  mark(MOGA_STAGE_STGA_ATTN, false, c.stream);
  count(1);
  return from_cuda(e);
}

// ------------------------------------------------------------------ training
struct BwdWs {
  size_t table, permw, qh, kh, vh, doh, dsum, dgate, route, total;
};
BwdWs bwd_ws(int64_t N, int d, int H, int d_h, int M) {
  Carve c;
  BwdWs w;
  const size_t mat = (size_t)N * H * d_h * 2;
  w.table = c.take((size_t)(3 * M + 1) * 4);
  w.permw = c.take((size_t)N * 4);
  w.qh = c.take(mat);
  w.kh = c.take(mat);
  w.vh = c.take(mat);
  w.doh = c.take(mat);
  w.dsum = c.take((size_t)N * H * 4);
  w.dgate = c.take((size_t)N * 4);
  w.route = c.take(route_bwd_ws_bytes(N, d, M));
  w.total = c.off;
  return w;
}

// One branch of the attention backward: dO and D, then dK/dV, then dQ.
// mode 0: groups (perm, offsets, gate); mode 1: STGA windows (window order).
moga_status attn_bwd_branch(const DevCtx& c, const BwdWs& w, uint8_t* ws, int mode, const void* dout, const void* o,
                            const float* lse, const void* q, const void* k, const void* v, const int32_t* perm,
                            const int32_t* offsets, const float* gate, float wgt, int64_t N, int H, int d_h, int M,
                            int T, int Hg, int Wg, const int* window, int accumulate, void* dq, void* dk, void* dv) {
  int32_t* table = reinterpret_cast<int32_t*>(ws + w.table);
  int32_t* permw = reinterpret_cast<int32_t*>(ws + w.permw);
  float* dsum = reinterpret_cast<float*>(ws + w.dsum);
  float* dgate = reinterpret_cast<float*>(ws + w.dgate);
  const int32_t* sp = perm;
  if (mode == 0) {
    if (launch_seg_table(c, offsets, M, H, N, table, 1) != cudaSuccess) return MOGA_ERR_CUDA;
  } else {
    if (launch_window_perm(c, T, Hg, Wg, window, permw) != cudaSuccess) return MOGA_ERR_CUDA;
    sp = permw;
  }
  if (launch_gather(c, q, k, v, sp, N, H, d_h, ws + w.qh, ws + w.kh, ws + w.vh) != cudaSuccess) return MOGA_ERR_CUDA;
  if (launch_bwd_prep(c, dout, o, sp, mode == 0 ? gate : nullptr, wgt, N, H, d_h, ws + w.doh, dsum,
                      mode == 0 ? dgate : nullptr) != cudaSuccess)
    return MOGA_ERR_CUDA;
  count(3);
  BwdArgs a{};
  a.q = ws + w.qh;
  a.k = ws + w.kh;
  a.v = ws + w.vh;
  a.dout = ws + w.doh;
  a.lse = lse;
  a.dsum = dsum;
  a.perm = sp;
  a.N = N;
  a.H = H;
  a.d_h = d_h;
  a.accumulate = accumulate;
  a.mode = mode;
  if (mode == 0) {
    a.table = table;
    a.nseg = M;
  } else {
    a.nseg = (int)stga_num_windows(T, Hg, Wg, window);
    a.T = T;
    a.Hg = Hg;
    a.Wg = Wg;
    a.wt = window[0];
    a.wh = window[1];
    a.ww = window[2];
  }
  a.out1 = dv;
  a.out2 = dk;
  if (launch_attn_bwd(c, a, false) != cudaSuccess) return MOGA_ERR_CUDA;
  a.out1 = dq;
  a.out2 = nullptr;
  if (launch_attn_bwd(c, a, true) != cudaSuccess) return MOGA_ERR_CUDA;
  count(2);
  return MOGA_OK;
}

moga_status check_route_args(const void* x, const void* W_r, const float* b_r, moga_dtype dt, int64_t N, int d,
                             int M, const int32_t* gid, const float* gate, const int32_t* perm,
                             const int32_t* offsets, const int32_t* max_seqlen) {
  if (N < 0 || N >= ((int64_t)1 << 31) || M < 1 || M > 1024) return MOGA_ERR_INVALID_ARG;
  // per-token buffers may be NULL when there are no tokens
  if (!W_r || !offsets || !max_seqlen || (N > 0 && (!x || !gid || !gate || !perm))) return MOGA_ERR_INVALID_ARG;
  if (dt != MOGA_F32 && dt != MOGA_BF16) return MOGA_ERR_INVALID_ARG;
  if (d < 1) return MOGA_ERR_INVALID_ARG;
  if (dt == MOGA_BF16 && (d % 8) != 0) return MOGA_ERR_UNSUPPORTED;
  if (dt == MOGA_F32 && (d % 4) != 0) return MOGA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(W_r)) return MOGA_ERR_INVALID_ARG;
  if ((b_r && !aligned4(b_r)) || !aligned4(gid) || !aligned4(gate) || !aligned4(perm) || !aligned4(offsets) ||
      !aligned4(max_seqlen))
    return MOGA_ERR_INVALID_ARG;
  return MOGA_OK;
}

// q, k, v and out may be NULL only when there are no tokens (n == 0).
moga_status check_qkv(const void* q, const void* k, const void* v, const void* out, int64_t n = 1) {
  if (n > 0 && (!q || !k || !v || !out)) return MOGA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return MOGA_ERR_INVALID_ARG;
  return MOGA_OK;
}

// Shot windows whose key/value segments span at most four tiles are read in
// place; longer ones (the pages' whole-shot windows) stream each K/V tile for
// many query tiles and read gathered head-major copies with tiled loads.
bool shot_direct(int T, int Hg, int Wg, const int* w, int nshots, int aug_prev, int aug_next) {
  const int64_t frames = (int64_t)(w[0] > 0 ? w[0] : T - nshots + 1) + aug_prev + aug_next;
  const int64_t area = (int64_t)(w[1] < Hg ? w[1] : Hg) * (w[2] < Wg ? w[2] : Wg);
  return frames * area <= 4 * kTile;
}

// Shot windows: window table, query index list, key/value index list, and
// (tiled) the gathered copies of Q (N rows per head) and K/V (kv_cap rows).
struct ShotWs {
  size_t wtab, qperm, kvperm, qh, kh, vh, total;
  int64_t cap, kv_cap;
  bool direct;
};
ShotWs shot_ws(int T, int Hg, int Wg, const int* window, int nshots, int aug_prev, int aug_next, int H, int d_h) {
  Carve c;
  ShotWs w;
  const int64_t N = (int64_t)T * Hg * Wg;
  w.cap = shot_window_cap(T, Hg, Wg, window, nshots);
  w.kv_cap = shot_kv_cap(T, Hg, Wg, nshots, aug_prev, aug_next);
  w.direct = shot_direct(T, Hg, Wg, window, nshots, aug_prev, aug_next);
  w.wtab = c.take(shot_table_ints(w.cap) * 4);
  w.qperm = c.take((size_t)N * 4);
  w.kvperm = c.take((size_t)w.kv_cap * 4);
  w.qh = w.kh = w.vh = 0;
  if (!w.direct) {
    w.qh = c.take((size_t)N * H * d_h * 2);
    w.kh = c.take((size_t)w.kv_cap * H * d_h * 2);
    w.vh = c.take((size_t)w.kv_cap * H * d_h * 2);
  }
  w.total = c.off;
  return w;
}

moga_status check_shots(int T, int Hg, int Wg, const int* window, int nshots, int aug_prev, int aug_next,
                        int64_t* N) {
  if (!window || T < 1 || Hg < 1 || Wg < 1) return MOGA_ERR_INVALID_ARG;
  if (window[0] < 0 || window[1] < 1 || window[2] < 1) return MOGA_ERR_INVALID_ARG;
  if (nshots < 1 || nshots > T || aug_prev < 0 || aug_next < 0 || aug_prev > T || aug_next > T)
    return MOGA_ERR_INVALID_ARG;
  const int64_t n = (int64_t)T * Hg * Wg;
  if (n >= (int64_t)1 << 31 || shot_kv_cap(T, Hg, Wg, nshots, aug_prev, aug_next) >= (int64_t)1 << 30 ||
      (int64_t)shot_table_ints(shot_window_cap(T, Hg, Wg, window, nshots)) >= (int64_t)1 << 31)
    return MOGA_ERR_UNSUPPORTED;
  *N = n;
  return MOGA_OK;
}

moga_status check_shot_args(int T, int Hg, int Wg, const int* window, const int32_t* shot_start, int nshots,
                            int aug_prev, int aug_next, int H, int d_h, int64_t* N) {
  moga_status st = check_shots(T, Hg, Wg, window, nshots, aug_prev, aug_next, N);
  if (st != MOGA_OK) return st;
  if ((st = check_attn_shape(*N, H, d_h)) != MOGA_OK) return st;
  if (!shot_start || !aligned4(shot_start)) return MOGA_ERR_INVALID_ARG;
  if ((int64_t)shot_kv_cap(T, Hg, Wg, nshots, aug_prev, aug_next) * H >= (int64_t)1 << 31)
    return MOGA_ERR_UNSUPPORTED;
  return MOGA_OK;
}

// Shot-aware STGA into out (accumulate: out += out_scale * SA), arguments
// already validated, workspace large enough for shot_ws.
moga_status shot_body(const DevCtx& c, const void* q, const void* k, const void* v, int T, int Hg, int Wg,
                      const int* window, const int32_t* shot_start, int nshots, int aug_prev, int aug_next, int H,
                      int d_h, float out_scale, int accumulate, void* out, uint8_t* wb) {
  const int64_t N = (int64_t)T * Hg * Wg;
  const ShotWs w = shot_ws(T, Hg, Wg, window, nshots, aug_prev, aug_next, H, d_h);
  int32_t* wtab = reinterpret_cast<int32_t*>(wb + w.wtab);
  int32_t* qperm = reinterpret_cast<int32_t*>(wb + w.qperm);
  int32_t* kvperm = reinterpret_cast<int32_t*>(wb + w.kvperm);
  mark(MOGA_STAGE_STGA_PREP, true, c.stream);
  if (launch_shot_table(c, shot_start, nshots, T, Hg, Wg, window, aug_prev, aug_next, H, w.cap, wtab) !=
      cudaSuccess)
    return MOGA_ERR_CUDA;
  if (launch_shot_perm(c, wtab, w.cap, Hg, Wg, window, qperm, kvperm) != cudaSuccess) return MOGA_ERR_CUDA;
  count(2);
  AttnArgs a{};
  a.direct = w.direct ? 1 : 0;
  a.q = q;
  a.k = k;
  a.v = v;
  if (!w.direct) {
    // queries: every token once; keys/values: the device-computed count of rows
    if (launch_gather_rows(c, q, nullptr, qperm, nullptr, N, N, H, d_h, N, wb + w.qh, nullptr) != cudaSuccess ||
        launch_gather_rows(c, k, v, kvperm, wtab + 2, w.kv_cap, N, H, d_h, w.kv_cap, wb + w.kh, wb + w.vh) !=
            cudaSuccess)
      return MOGA_ERR_CUDA;
    count(2);
    a.q = wb + w.qh;
    a.k = wb + w.kh;
    a.v = wb + w.vh;
    a.kv_rows = w.kv_cap;
  }
  mark(MOGA_STAGE_STGA_PREP, false, c.stream);
  a.perm = qperm;
  a.kvperm = kvperm;
  a.gate = nullptr;
  a.out = out;
  a.N = N;
  a.H = H;
  a.d_h = d_h;
  a.out_scale = out_scale;
  a.accumulate = accumulate;
  a.mode = 2;
  a.table = wtab;
  a.nseg = (int)w.cap;
  a.T = T;
  a.Hg = Hg;
  a.Wg = Wg;
  a.wt = window[0];
  a.wh = window[1];
  a.ww = window[2];
  a.debug_withhold_first_k = g_debug_inject.load(std::memory_order_relaxed) == 1;
  mark(MOGA_STAGE_STGA_ATTN, true, c.stream);
  const cudaError_t e = launch_attention(c, a);
  mark(MOGA_STAGE_STGA_ATTN, false, c.stream);
  count(1);
  return from_cuda(e);
}

}  // namespace

bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                  uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_box5(CUtensorMap* map, const void* base, uint64_t d_h, uint64_t H, uint64_t Wg, uint64_t Hg,
                    uint64_t T, const int* window) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[5] = {d_h, H, Wg, Hg, T};
  cuuint64_t strides[4] = {d_h * 2, H * d_h * 2, Wg * H * d_h * 2, Hg * Wg * H * d_h * 2};
  cuuint32_t box[5] = {64, 1, (cuuint32_t)window[2], (cuuint32_t)window[1], (cuuint32_t)window[0]};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  for (int i = 2; i < 5; ++i)
    if (box[i] < 1 || box[i] > 256) return false;
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_tokens(CUtensorMap* map, const void* base, uint64_t d_h, uint64_t H, uint64_t N) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d_h, H, N};
  cuuint64_t strides[2] = {d_h * 2, H * d_h * 2};
  cuuint32_t box[3] = {64, 1, (cuuint32_t)kTile};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace moga

using namespace moga;

extern "C" {

const char* moga_status_string(int s) {
  switch (s) {
    case MOGA_OK: return "MOGA_OK";
    case MOGA_ERR_INVALID_ARG: return "MOGA_ERR_INVALID_ARG";
    case MOGA_ERR_UNSUPPORTED: return "MOGA_ERR_UNSUPPORTED";
    case MOGA_ERR_WORKSPACE: return "MOGA_ERR_WORKSPACE";
    case MOGA_ERR_CUDA: return "MOGA_ERR_CUDA";
    case MOGA_ERR_TIMEOUT: return "MOGA_ERR_TIMEOUT";
    case MOGA_ERR_DEVICE_CHECK: return "MOGA_ERR_DEVICE_CHECK";
    default: return "MOGA_ERR_UNKNOWN";
  }
}

int moga_version(void) { return (1 << 16) | 0; }

uint64_t moga_set_wait_limit_ns(uint64_t ns) { return g_wait_ns.exchange(ns ? ns : 1); }

uint64_t moga_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

moga_status moga_debug_inject(int mode) {
  if (mode < 0 || mode > 1) return MOGA_ERR_INVALID_ARG;
  g_debug_inject.store(mode, std::memory_order_relaxed);
  return MOGA_OK;
}

moga_status moga_set_timing_events(int stage, void* begin, void* end) {
  if (stage < 0 || stage >= kNumStages) return MOGA_ERR_INVALID_ARG;
  if ((begin == nullptr) != (end == nullptr)) return MOGA_ERR_INVALID_ARG;
  g_ev_begin[stage].store(begin, std::memory_order_relaxed);
  g_ev_end[stage].store(end, std::memory_order_relaxed);
  return MOGA_OK;
}

size_t moga_route_workspace_size(int64_t N, int M) {
  if (N < 0 || M < 1) return 0;
  return route_ws(N, M).total;
}

moga_status moga_route(const void* x, const void* W_r, const float* b_r, moga_dtype dt, int64_t N, int d, int M,
                       int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets, int32_t* max_seqlen,
                       void* ws, size_t ws_bytes, void* stream) {
  moga_status st = check_route_args(x, W_r, b_r, dt, N, d, M, group_id, gate, perm, offsets, max_seqlen);
  if (st != MOGA_OK) return st;
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < route_ws(N, M).total) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  return route_body(c, x, W_r, b_r, dt, N, d, M, group_id, gate, perm, offsets, max_seqlen, (uint8_t*)ws);
}

size_t moga_sort_workspace_size(int64_t N, int M) {
  if (N < 0 || M < 1) return 0;
  return route_ws(N, M).total;
}

moga_status moga_sort(const int32_t* group_id, int64_t N, int M, int32_t* perm, int32_t* offsets,
                      int32_t* max_seqlen, void* ws, size_t ws_bytes, void* stream) {
  // scan_kernel keeps one shared-memory slot per group in 1024-entry arrays
  // and sums each group with one of its 1024 threads, so M is capped there.
  if (N < 0 || N >= ((int64_t)1 << 31) || M < 1 || M > 1024) return MOGA_ERR_INVALID_ARG;
  if (!offsets || !max_seqlen || !aligned4(offsets) || !aligned4(max_seqlen)) return MOGA_ERR_INVALID_ARG;
  if (N > 0 && (!group_id || !perm || !aligned4(group_id) || !aligned4(perm))) return MOGA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < moga_sort_workspace_size(N, M)) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  if (N == 0) {
    cudaError_t e = cudaMemsetAsync(offsets, 0, (size_t)(M + 1) * 4, c.stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(max_seqlen, 0, 4, c.stream);
    return from_cuda(e);
  }
  const RouteWs w = route_ws(N, M);
  int32_t* hist = reinterpret_cast<int32_t*>((uint8_t*)ws + w.hist);
  int32_t* base = reinterpret_cast<int32_t*>((uint8_t*)ws + w.base);
  mark(MOGA_STAGE_SORT, true, c.stream);
  if (launch_hist(c, group_id, N, M, hist) != cudaSuccess ||
      launch_scan(c, hist, ceil_div(N, kTile), M, base, offsets, max_seqlen, nullptr, N, nullptr, nullptr) !=
          cudaSuccess ||
      launch_scatter(c, group_id, base, N, M, perm) != cudaSuccess)
    return MOGA_ERR_CUDA;
  mark(MOGA_STAGE_SORT, false, c.stream);
  count(3);
  return MOGA_OK;
}

size_t moga_route_ex_workspace_size(int64_t N, int M) {
  if (N < 0 || M < 1) return 0;
  return route_ws(N, M, true).total;
}

moga_status moga_route_ex(const void* x, const void* W_r, const float* b_r, moga_dtype dt, int64_t N, int d, int M,
                          int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets, int32_t* max_seqlen,
                          float* prob_mean, float* balance, void* ws, size_t ws_bytes, void* stream) {
  moga_status st = check_route_args(x, W_r, b_r, dt, N, d, M, group_id, gate, perm, offsets, max_seqlen);
  if (st != MOGA_OK) return st;
  if ((prob_mean && !aligned4(prob_mean)) || (balance && !aligned4(balance))) return MOGA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  const bool stats = prob_mean || balance;
  if (ws_bytes < route_ws(N, M, stats).total) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  return route_body(c, x, W_r, b_r, dt, N, d, M, group_id, gate, perm, offsets, max_seqlen, (uint8_t*)ws,
                    prob_mean, balance);
}

moga_status moga_route_noalloc(const void* x, const void* W_r, const float* b_r, moga_dtype dt, int64_t N, int d,
                               int M, int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets,
                               int32_t* max_seqlen, void* stream) {
  moga_status st = check_route_args(x, W_r, b_r, dt, N, d, M, group_id, gate, perm, offsets, max_seqlen);
  if (st != MOGA_OK) return st;
  if (ceil_div(N, kTile) * (int64_t)M > kNoAllocCells) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, nullptr, stream)) return MOGA_ERR_CUDA;
  uint8_t* scratch = noalloc_scratch(c.device);
  if (!scratch) return MOGA_ERR_CUDA;
  c.status = reinterpret_cast<int*>(scratch);
  // route_body writes every scratch word it reads later, except the tile
  // histogram of the tensor-core router, which its launcher zeroes first.
  return route_body(c, x, W_r, b_r, dt, N, d, M, group_id, gate, perm, offsets, max_seqlen, scratch);
}

size_t moga_group_attn_workspace_size(int64_t N, int H, int d_h, int M) {
  if (N < 0 || H < 1 || M < 1) return 0;
  return attn_ws(N, H, d_h, M, false).total;
}

moga_status moga_group_attn(const void* q, const void* k, const void* v, const int32_t* perm,
                            const int32_t* offsets, const float* gate, int64_t N, int H, int d_h, int M,
                            float out_scale, void* out, void* ws, size_t ws_bytes, void* stream) {
  moga_status st = check_qkv(q, k, v, out, N);
  if (st != MOGA_OK) return st;
  if (!perm || !offsets || !aligned4(perm) || !aligned4(offsets) || (gate && !aligned4(gate)))
    return MOGA_ERR_INVALID_ARG;
  if (M < 1 || M > 1024) return MOGA_ERR_INVALID_ARG;
  if ((st = check_attn_shape(N, H, d_h)) != MOGA_OK) return st;
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < attn_ws(N, H, d_h, M, false).total) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  return group_attn_body(c, q, k, v, perm, offsets, gate, N, H, d_h, M, out_scale, out, (uint8_t*)ws);
}

size_t stga_window_attn_workspace_size(int T, int Hg, int Wg, const int* window, int H, int d_h) {
  int64_t N = 0;
  if (check_window(T, Hg, Wg, window, &N) != MOGA_OK || H < 1) return 0;
  return attn_ws(N, H, d_h, 0, true, !stga_direct(window)).total;
}

moga_status stga_window_attn(const void* q, const void* k, const void* v, int T, int Hg, int Wg,
                             const int* window, int H, int d_h, int accumulate, void* out, void* ws,
                             size_t ws_bytes, void* stream) {
  moga_status st = check_qkv(q, k, v, out);
  if (st != MOGA_OK) return st;
  int64_t N = 0;
  if ((st = check_window(T, Hg, Wg, window, &N)) != MOGA_OK) return st;
  if ((st = check_attn_shape(N, H, d_h)) != MOGA_OK) return st;
  if (accumulate != 0 && accumulate != 1) return MOGA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < attn_ws(N, H, d_h, 0, true, !stga_direct(window)).total) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  return stga_body(c, q, k, v, T, Hg, Wg, window, H, d_h, accumulate, out, (uint8_t*)ws);
}

size_t stga_shot_attn_workspace_size(int T, int Hg, int Wg, const int* window, int nshots, int aug_prev,
                                     int aug_next, int H, int d_h) {
  int64_t N = 0;
  if (check_shots(T, Hg, Wg, window, nshots, aug_prev, aug_next, &N) != MOGA_OK) return 0;
  if (check_attn_shape(N, H, d_h) != MOGA_OK) return 0;
  return shot_ws(T, Hg, Wg, window, nshots, aug_prev, aug_next, H, d_h).total;
}

moga_status stga_shot_attn(const void* q, const void* k, const void* v, int T, int Hg, int Wg, const int* window,
                           const int32_t* shot_start, int nshots, int aug_prev, int aug_next, int H, int d_h,
                           float out_scale, int accumulate, void* out, void* ws, size_t ws_bytes, void* stream) {
  moga_status st = check_qkv(q, k, v, out);
  if (st != MOGA_OK) return st;
  int64_t N = 0;
  if ((st = check_shot_args(T, Hg, Wg, window, shot_start, nshots, aug_prev, aug_next, H, d_h, &N)) != MOGA_OK)
    return st;
  if ((accumulate != 0 && accumulate != 1) || !(out_scale == out_scale)) return MOGA_ERR_INVALID_ARG;  // NaN
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < shot_ws(T, Hg, Wg, window, nshots, aug_prev, aug_next, H, d_h).total) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  return shot_body(c, q, k, v, T, Hg, Wg, window, shot_start, nshots, aug_prev, aug_next, H, d_h, out_scale,
                   accumulate, out, (uint8_t*)ws);
}

size_t moga_layer_shots_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg, const int* window,
                                       int nshots, int aug_prev, int aug_next, int per_frame) {
  if (N < 0 || H < 1 || M < 1 || (per_frame != 0 && per_frame != 1)) return 0;
  if (stga_shot_attn_workspace_size(T, Hg, Wg, window, nshots, aug_prev, aug_next, H, d_h) == 0) return 0;
  size_t need = moga_layer_ex_workspace_size(N, H, d_h, M, per_frame ? 2 : 0);
  const size_t sw = shot_ws(T, Hg, Wg, window, nshots, aug_prev, aug_next, H, d_h).total;
  return need > sw ? need : sw;
}

moga_status moga_layer_shots(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                             const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                             int Wg, const int* window, const int32_t* shot_start, int nshots, int aug_prev,
                             int aug_next, int per_frame, void* out, int32_t* group_id, float* gate, int32_t* perm,
                             int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  if (per_frame != 0 && per_frame != 1) return MOGA_ERR_INVALID_ARG;
  moga_status st = check_route_args(x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, offsets);
  if (st != MOGA_OK) return st;
  if ((st = check_qkv(q, k, v, out)) != MOGA_OK) return st;
  if ((st = check_attn_shape(N, H, d_h)) != MOGA_OK) return st;
  int64_t n = 0;
  if ((st = check_shot_args(T, Hg, Wg, window, shot_start, nshots, aug_prev, aug_next, H, d_h, &n)) != MOGA_OK)
    return st;
  if (n != N) return MOGA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < moga_layer_shots_workspace_size(N, H, d_h, M, T, Hg, Wg, window, nshots, aug_prev, aug_next,
                                                 per_frame))
    return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  uint8_t* w = (uint8_t*)ws;
  int32_t* max_seqlen = reinterpret_cast<int32_t*>(w + 16);
  if ((st = route_body(c, x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, max_seqlen, w)) != MOGA_OK)
    return st;
  if (N == 0) return MOGA_OK;
  // out = mean of MoGA, shot-aware STGA and (when on) the per-frame branch
  const float scale = 1.0f / (float)(2 + per_frame);
  const int frame_window[3] = {1, Hg, Wg};
  if ((st = group_attn_body(c, q, k, v, perm, offsets, gate, N, H, d_h, M, scale, out, w)) != MOGA_OK) return st;
  if ((st = shot_body(c, q, k, v, T, Hg, Wg, window, shot_start, nshots, aug_prev, aug_next, H, d_h, scale, 1, out,
                      w)) != MOGA_OK)
    return st;
  if (per_frame && (st = stga_body(c, q, k, v, T, Hg, Wg, frame_window, H, d_h, 1, out, w, scale)) != MOGA_OK)
    return st;
  return MOGA_OK;
}

size_t moga_layer_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg, const int* window) {
  if (N < 0 || H < 1 || M < 1) return 0;
  size_t need = route_ws(N, M).total;
  const size_t ga = attn_ws(N, H, d_h, M, false).total;
  if (ga > need) need = ga;
  if (window) {
    const size_t sw = attn_ws(N, H, d_h, 0, true, !stga_direct(window)).total;
    if (sw > need) need = sw;
  }
  return need;
}

moga_status moga_layer(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                       const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                       int Wg, const int* window, void* out, int32_t* group_id, float* gate, int32_t* perm,
                       int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  moga_status st = check_route_args(x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, offsets);
  if (st != MOGA_OK) return st;
  if ((st = check_qkv(q, k, v, out, N)) != MOGA_OK) return st;
  if ((st = check_attn_shape(N, H, d_h)) != MOGA_OK) return st;
  if (window) {
    int64_t n = 0;
    if ((st = check_window(T, Hg, Wg, window, &n)) != MOGA_OK) return st;
    if (n != N) return MOGA_ERR_INVALID_ARG;
  }
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < moga_layer_workspace_size(N, H, d_h, M, T, Hg, Wg, window)) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  uint8_t* w = (uint8_t*)ws;
  // max_seqlen has no output slot in the layer call: keep it in the header.
  int32_t* max_seqlen = reinterpret_cast<int32_t*>(w + 16);
  if ((st = route_body(c, x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, max_seqlen, w)) != MOGA_OK)
    return st;
  if (N == 0) return MOGA_OK;
  const float scale = window ? 0.5f : 1.0f;
  if ((st = group_attn_body(c, q, k, v, perm, offsets, gate, N, H, d_h, M, scale, out, w)) != MOGA_OK) return st;
  if (window) return stga_body(c, q, k, v, T, Hg, Wg, window, H, d_h, 1, out, w);
  return MOGA_OK;
}

size_t moga_layer_train_ex_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg,
                                          const int* window, int per_frame) {
  if (per_frame != 0 && per_frame != 1) return 0;
  if (!per_frame) return moga_layer_workspace_size(N, H, d_h, M, T, Hg, Wg, window);
  return moga_layer_ex_workspace_size(N, H, d_h, M, (window ? 1 : 0) | 2);
}

size_t moga_layer_train_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg, const int* window) {
  return moga_layer_train_ex_workspace_size(N, H, d_h, M, T, Hg, Wg, window, 0);
}

moga_status moga_layer_train_ex(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                                const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                                int Wg, const int* window, int per_frame, void* out, void* o_moga, void* o_stga,
                                void* o_frame, float* lse_moga, float* lse_stga, float* lse_frame, int32_t* group_id,
                                float* gate, int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes,
                                void* stream) {
  if (per_frame != 0 && per_frame != 1) return MOGA_ERR_INVALID_ARG;
  moga_status st = check_route_args(x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, offsets);
  if (st != MOGA_OK) return st;
  if ((st = check_qkv(q, k, v, out, N)) != MOGA_OK) return st;
  if ((st = check_attn_shape(N, H, d_h)) != MOGA_OK) return st;
  if ((N > 0 && !o_moga) || !aligned16(o_moga) || (N > 0 && (!lse_moga || !aligned4(lse_moga))))
    return MOGA_ERR_INVALID_ARG;
  const int frame_window[3] = {1, Hg, Wg};
  if (window || per_frame) {
    int64_t n = 0;
    if ((st = check_window(T, Hg, Wg, window ? window : frame_window, &n)) != MOGA_OK) return st;
    if (n != N) return MOGA_ERR_INVALID_ARG;
    if (out == o_moga) return MOGA_ERR_INVALID_ARG;
  }
  if (window) {
    if (!o_stga || !aligned16(o_stga) || (N > 0 && (!lse_stga || !aligned4(lse_stga)))) return MOGA_ERR_INVALID_ARG;
    if (out == o_stga || o_moga == o_stga) return MOGA_ERR_INVALID_ARG;
  }
  if (per_frame) {
    if (!o_frame || !aligned16(o_frame) || (N > 0 && (!lse_frame || !aligned4(lse_frame))))
      return MOGA_ERR_INVALID_ARG;
    if (out == o_frame || o_moga == o_frame || (window && o_stga == o_frame)) return MOGA_ERR_INVALID_ARG;
  }
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < moga_layer_train_ex_workspace_size(N, H, d_h, M, T, Hg, Wg, window, per_frame))
    return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  uint8_t* w = (uint8_t*)ws;
  int32_t* max_seqlen = reinterpret_cast<int32_t*>(w + 16);
  if ((st = route_body(c, x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, max_seqlen, w)) != MOGA_OK)
    return st;
  if (N == 0) return MOGA_OK;
  if ((st = group_attn_body(c, q, k, v, perm, offsets, gate, N, H, d_h, M, 1.0f, o_moga, w, lse_moga)) != MOGA_OK)
    return st;
  const int64_t n = N * H * d_h;
  if (window &&
      (st = stga_body(c, q, k, v, T, Hg, Wg, window, H, d_h, 0, o_stga, w, 1.0f, lse_stga)) != MOGA_OK)
    return st;
  if (per_frame &&
      (st = stga_body(c, q, k, v, T, Hg, Wg, frame_window, H, d_h, 0, o_frame, w, 1.0f, lse_frame)) != MOGA_OK)
    return st;
  if (window || per_frame) {
    // out = the plain mean of the branches that are on
    const void* b2 = window ? o_stga : o_frame;
    const void* b3 = (window && per_frame) ? o_frame : nullptr;
    if (launch_mean(c, o_moga, b2, b3, n, out) != cudaSuccess) return MOGA_ERR_CUDA;
    count(1);
  } else if (out != o_moga) {
    if (cudaMemcpyAsync(out, o_moga, (size_t)n * 2, cudaMemcpyDeviceToDevice, c.stream) != cudaSuccess)
      return MOGA_ERR_CUDA;
  }
  return MOGA_OK;
}

moga_status moga_layer_train(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                             const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                             int Wg, const int* window, void* out, void* o_moga, void* o_stga, float* lse_moga,
                             float* lse_stga, int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets,
                             void* ws, size_t ws_bytes, void* stream) {
  return moga_layer_train_ex(x, W_r, b_r, x_dt, q, k, v, N, d, H, d_h, M, T, Hg, Wg, window, 0, out, o_moga, o_stga,
                             nullptr, lse_moga, lse_stga, nullptr, group_id, gate, perm, offsets, ws, ws_bytes,
                             stream);
}

size_t moga_layer_backward_workspace_size(int64_t N, int d, int H, int d_h, int M) {
  if (N < 0 || d < 1 || H < 1 || M < 1 || M > 1024 || (d_h != 64 && d_h != 128)) return 0;
  return bwd_ws(N, d, H, d_h, M).total;
}

moga_status moga_layer_backward_ex(const void* dout, const void* x, const void* W_r, const float* b_r,
                                   moga_dtype x_dt, const void* q, const void* k, const void* v, int64_t N, int d,
                                   int H, int d_h, int M, int T, int Hg, int Wg, const int* window, int per_frame,
                                   float balance_alpha, const void* o_moga, const void* o_stga, const void* o_frame,
                                   const float* lse_moga,
                                   const float* lse_stga, const float* lse_frame, const int32_t* group_id,
                                   const float* gate, const int32_t* perm, const int32_t* offsets, void* dx,
                                   float* dW_r, float* db_r, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                   void* stream) {
  if (per_frame != 0 && per_frame != 1) return MOGA_ERR_INVALID_ARG;
  if (!std::isfinite(balance_alpha))
    return MOGA_ERR_INVALID_ARG;
  // the routing results are inputs here; the forward's checks cover them
  moga_status st = check_route_args(x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, offsets);
  if (st != MOGA_OK) return st;
  if ((st = check_qkv(q, k, v, dout, N)) != MOGA_OK) return st;
  if ((st = check_attn_shape(N, H, d_h)) != MOGA_OK) return st;
  if ((st = check_qkv(dq, dk, dv, o_moga, N)) != MOGA_OK) return st;
  if (!dW_r || !aligned4(dW_r) || (db_r && !aligned4(db_r))) return MOGA_ERR_INVALID_ARG;
  if (N > 0 && (!dx || !aligned16(dx) || !lse_moga || !aligned4(lse_moga))) return MOGA_ERR_INVALID_ARG;
  const int frame_window[3] = {1, Hg, Wg};
  if (window || per_frame) {
    int64_t n = 0;
    if ((st = check_window(T, Hg, Wg, window ? window : frame_window, &n)) != MOGA_OK) return st;
    if (n != N) return MOGA_ERR_INVALID_ARG;
  }
  if (window && (!o_stga || !aligned16(o_stga) || (N > 0 && (!lse_stga || !aligned4(lse_stga)))))
    return MOGA_ERR_INVALID_ARG;
  if (per_frame && (!o_frame || !aligned16(o_frame) || (N > 0 && (!lse_frame || !aligned4(lse_frame)))))
    return MOGA_ERR_INVALID_ARG;
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < moga_layer_backward_workspace_size(N, d, H, d_h, M)) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  uint8_t* w = (uint8_t*)ws;
  const BwdWs bw = bwd_ws(N, d, H, d_h, M);
  if (N == 0) {
    cudaError_t e = cudaMemsetAsync(dW_r, 0, (size_t)M * d * 4, c.stream);
    if (e == cudaSuccess && db_r) e = cudaMemsetAsync(db_r, 0, (size_t)M * 4, c.stream);
    return from_cuda(e);
  }
  // each branch's share of dout: one over the number of branches
  const float wgt = 1.0f / (float)(1 + (window ? 1 : 0) + per_frame);
  if ((st = attn_bwd_branch(c, bw, w, 0, dout, o_moga, lse_moga, q, k, v, perm, offsets, gate, wgt, N, H, d_h, M,
                            T, Hg, Wg, window, 0, dq, dk, dv)) != MOGA_OK)
    return st;
  if (window && (st = attn_bwd_branch(c, bw, w, 1, dout, o_stga, lse_stga, q, k, v, nullptr, nullptr, nullptr, wgt,
                                      N, H, d_h, M, T, Hg, Wg, window, 1, dq, dk, dv)) != MOGA_OK)
    return st;
  if (per_frame && (st = attn_bwd_branch(c, bw, w, 1, dout, o_frame, lse_frame, q, k, v, nullptr, nullptr, nullptr,
                                         wgt, N, H, d_h, M, T, Hg, Wg, frame_window, 1, dq, dk, dv)) != MOGA_OK)
    return st;
  if (launch_route_bwd(c, x, W_r, b_r, x_dt == MOGA_BF16, N, d, M, group_id,
                       reinterpret_cast<const float*>(w + bw.dgate), offsets, balance_alpha, dx, dW_r, db_r,
                       w + bw.route) != cudaSuccess)
    return MOGA_ERR_CUDA;
  count(3);
  return MOGA_OK;
}

moga_status moga_layer_backward(const void* dout, const void* x, const void* W_r, const float* b_r, moga_dtype x_dt,
                                const void* q, const void* k, const void* v, int64_t N, int d, int H, int d_h, int M,
                                int T, int Hg, int Wg, const int* window, const void* o_moga, const void* o_stga,
                                const float* lse_moga, const float* lse_stga, const int32_t* group_id,
                                const float* gate, const int32_t* perm, const int32_t* offsets, void* dx,
                                float* dW_r, float* db_r, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                void* stream) {
  return moga_layer_backward_ex(dout, x, W_r, b_r, x_dt, q, k, v, N, d, H, d_h, M, T, Hg, Wg, window, 0, 0.0f,
                                o_moga, o_stga, nullptr, lse_moga, lse_stga, nullptr, group_id, gate, perm, offsets,
                                dx, dW_r, db_r, dq, dk, dv, ws, ws_bytes, stream);
}

size_t moga_layer_ex_workspace_size(int64_t N, int H, int d_h, int M, int branches) {
  if (N < 0 || H < 1 || M < 1 || branches < 0 || branches > 3) return 0;
  size_t need = route_ws(N, M).total;
  const size_t ga = attn_ws(N, H, d_h, M, false).total;
  if (ga > need) need = ga;
  if (branches) {
    const size_t sw = attn_ws(N, H, d_h, 0, true).total;
    if (sw > need) need = sw;
  }
  return need;
}

moga_status moga_layer_ex(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                          const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                          int Wg, const int* window, int branches, void* out, int32_t* group_id, float* gate,
                          int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
  if (branches < 0 || branches > 3) return MOGA_ERR_INVALID_ARG;
  moga_status st = check_route_args(x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, offsets);
  if (st != MOGA_OK) return st;
  if ((st = check_qkv(q, k, v, out, N)) != MOGA_OK) return st;
  if ((st = check_attn_shape(N, H, d_h)) != MOGA_OK) return st;
  const int frame_window[3] = {1, Hg, Wg};
  if (branches & 1) {
    int64_t n = 0;
    if ((st = check_window(T, Hg, Wg, window, &n)) != MOGA_OK) return st;
    if (n != N) return MOGA_ERR_INVALID_ARG;
  }
  if (branches & 2) {
    int64_t n = 0;
    if ((st = check_window(T, Hg, Wg, frame_window, &n)) != MOGA_OK) return st;
    if (n != N) return MOGA_ERR_INVALID_ARG;
  }
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  if (ws_bytes < moga_layer_ex_workspace_size(N, H, d_h, M, branches)) return MOGA_ERR_WORKSPACE;
  DevCtx c;
  if (!make_ctx(&c, ws, stream)) return MOGA_ERR_CUDA;
  uint8_t* w = (uint8_t*)ws;
  int32_t* max_seqlen = reinterpret_cast<int32_t*>(w + 16);
  if ((st = route_body(c, x, W_r, b_r, x_dt, N, d, M, group_id, gate, perm, offsets, max_seqlen, w)) != MOGA_OK)
    return st;
  if (N == 0) return MOGA_OK;
  // out = mean of the branches that are on: each adds 1/nb of its output.
  const int nb = 1 + (branches & 1) + ((branches >> 1) & 1);
  const float scale = 1.0f / (float)nb;
  if ((st = group_attn_body(c, q, k, v, perm, offsets, gate, N, H, d_h, M, scale, out, w)) != MOGA_OK) return st;
  if ((branches & 1) && (st = stga_body(c, q, k, v, T, Hg, Wg, window, H, d_h, 1, out, w, scale)) != MOGA_OK)
    return st;
  if ((branches & 2) && (st = stga_body(c, q, k, v, T, Hg, Wg, frame_window, H, d_h, 1, out, w, scale)) != MOGA_OK)
    return st;
  return MOGA_OK;
}

moga_status moga_route_noalloc_status(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOGA_ERR_CUDA;
  uint8_t* scratch = noalloc_scratch(dev);
  if (!scratch) return MOGA_ERR_CUDA;
  return moga_sync_status(scratch, stream);
}

moga_status moga_sync_status(void* ws, void* stream) {
  if (!ws || !aligned16(ws)) return MOGA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOGA_ERR_CUDA;
  int word = 0;
  if (cudaMemcpy(&word, ws, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MOGA_ERR_CUDA;
  if (word != 0 && cudaMemset(ws, 0, sizeof(int)) != cudaSuccess) return MOGA_ERR_CUDA;
  if (word & DEV_TIMEOUT) return MOGA_ERR_TIMEOUT;
  if (word) return MOGA_ERR_DEVICE_CHECK;
  return MOGA_OK;
}

}  // extern "C"
