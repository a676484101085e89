// Host pipeline for the visual block of "MoGA: Mixture-of-Groups Attention for
// End-to-End Long Video Generation" (§3.4: MoGA, Eq. 5, plus the STGA and
// per-frame branches): the block runs on host-resident inputs and returns its
// output to host memory, with three streams so that consecutive steps overlap.
//
//   copy-in stream   H2D of step i+1's inputs into slot (i+1) % 2
//   compute stream   moga_layer_ex on slot i % 2 (router, sort, attention, ...)
//   copy-out stream  D2H of step i-1's outputs from slot (i-1) % 2
//
// Events order the slots: a slot's inputs are overwritten only after the step
// two back finished computing on them, and its outputs only after that step's
// copy-out finished.  The compute stream runs the steps in order, so one
// workspace (and one perm / offsets pair) serves both slots.
#include <cuda_runtime.h>

#include <cstdint>
#include <new>

#include "../../include/moga.h"

struct moga_pipe {
  struct Slot {
    void* x = nullptr;
    void* w = nullptr;
    float* b = nullptr;
    void* q = nullptr;
    void* k = nullptr;
    void* v = nullptr;
    void* out = nullptr;
    int32_t* gid = nullptr;
    float* gate = nullptr;
    cudaEvent_t in_done = nullptr, comp_done = nullptr, out_done = nullptr;
    bool used = false;
  };
  int dev = 0;
  int64_t N = 0;
  int d = 0, H = 0, d_h = 0, M = 0, T = 0, Hg = 0, Wg = 0, branches = 0;
  int window[3] = {0, 0, 0};
  bool has_window = false;
  moga_dtype x_dt = MOGA_BF16;
  size_t x_bytes = 0, w_bytes = 0, b_bytes = 0, qkv_bytes = 0, tok_bytes = 0, ws_bytes = 0;
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  Slot slot[2];
  int32_t* perm = nullptr;
  int32_t* offsets = nullptr;
  void* ws = nullptr;
  uint64_t steps = 0;
  moga_status err = MOGA_OK;  // first enqueue failure since the last sync
};

namespace {

// Makes the pipeline's device current for the scope of one call.
struct DeviceScope {
  int prev = -1;
  bool ok = false;
  explicit DeviceScope(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = prev == dev || cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceScope() {
    int cur = -1;
    if (prev >= 0 && cudaGetDevice(&cur) == cudaSuccess && cur != prev) cudaSetDevice(prev);
  }
};

// Device allocation of at least 16 bytes (so that empty shapes still get a
// valid, aligned pointer).
bool dalloc(void** p, size_t bytes) { return cudaMalloc(p, bytes < 16 ? 16 : bytes) == cudaSuccess; }

void release(moga_pipe* p) {
  if (p->s_in) cudaStreamSynchronize(p->s_in);
  if (p->s_comp) cudaStreamSynchronize(p->s_comp);
  if (p->s_out) cudaStreamSynchronize(p->s_out);
  for (auto& s : p->slot) {
    for (void* ptr : {s.x, s.w, static_cast<void*>(s.b), s.q, s.k, s.v, s.out, static_cast<void*>(s.gid),
                      static_cast<void*>(s.gate)})
      if (ptr) cudaFree(ptr);
    for (cudaEvent_t e : {s.in_done, s.comp_done, s.out_done})
      if (e) cudaEventDestroy(e);
  }
  if (p->perm) cudaFree(p->perm);
  if (p->offsets) cudaFree(p->offsets);
  if (p->ws) cudaFree(p->ws);
  for (cudaStream_t s : {p->s_in, p->s_comp, p->s_out})
    if (s) cudaStreamDestroy(s);
  delete p;
}

}  // namespace

extern "C" {

moga_status moga_pipe_create(int64_t N, int d, int H, int d_h, int M, moga_dtype x_dt, int T, int Hg, int Wg,
                             const int* window, int branches, moga_pipe** pipe) {
  if (!pipe) return MOGA_ERR_INVALID_ARG;
  *pipe = nullptr;
  if (N < 0 || N > INT32_MAX || d < 1 || H < 1 || M < 1 || branches < 0 || branches > 3) return MOGA_ERR_INVALID_ARG;
  if (x_dt != MOGA_F32 && x_dt != MOGA_BF16) return MOGA_ERR_INVALID_ARG;
  if (d_h != 64 && d_h != 128) return MOGA_ERR_UNSUPPORTED;
  if (branches) {
    if (T < 1 || Hg < 1 || Wg < 1 || (int64_t)T * Hg * Wg != N) return MOGA_ERR_INVALID_ARG;
    if ((branches & 1) && (!window || window[0] < 1 || window[1] < 1 || window[2] < 1)) return MOGA_ERR_INVALID_ARG;
  }
  const size_t ws_bytes = moga_layer_ex_workspace_size(N, H, d_h, M, branches);
  if (ws_bytes == 0) return MOGA_ERR_INVALID_ARG;

  moga_pipe* p = new (std::nothrow) moga_pipe();
  if (!p) return MOGA_ERR_CUDA;
  if (cudaGetDevice(&p->dev) != cudaSuccess) {
    delete p;
    return MOGA_ERR_CUDA;
  }
  p->N = N;
  p->d = d;
  p->H = H;
  p->d_h = d_h;
  p->M = M;
  p->x_dt = x_dt;
  p->T = T;
  p->Hg = Hg;
  p->Wg = Wg;
  p->branches = branches;
  p->has_window = (branches & 1) != 0;
  if (p->has_window)
    for (int i = 0; i < 3; ++i) p->window[i] = window[i];
  const size_t xe = x_dt == MOGA_F32 ? 4 : 2;
  p->x_bytes = (size_t)N * d * xe;
  p->w_bytes = (size_t)M * d * xe;
  p->b_bytes = (size_t)M * 4;
  p->qkv_bytes = (size_t)N * H * d_h * 2;
  p->tok_bytes = (size_t)N * 4;
  p->ws_bytes = ws_bytes;

  bool ok = cudaStreamCreateWithFlags(&p->s_in, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->s_comp, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&p->s_out, cudaStreamNonBlocking) == cudaSuccess;
  for (auto& s : p->slot) {
    ok = ok && dalloc(&s.x, p->x_bytes) && dalloc(&s.w, p->w_bytes) &&
         dalloc(reinterpret_cast<void**>(&s.b), p->b_bytes) && dalloc(&s.q, p->qkv_bytes) &&
         dalloc(&s.k, p->qkv_bytes) && dalloc(&s.v, p->qkv_bytes) && dalloc(&s.out, p->qkv_bytes) &&
         dalloc(reinterpret_cast<void**>(&s.gid), p->tok_bytes) &&
         dalloc(reinterpret_cast<void**>(&s.gate), p->tok_bytes);
    ok = ok && cudaEventCreateWithFlags(&s.in_done, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&s.comp_done, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&s.out_done, cudaEventDisableTiming) == cudaSuccess;
  }
  ok = ok && dalloc(reinterpret_cast<void**>(&p->perm), p->tok_bytes) &&
       dalloc(reinterpret_cast<void**>(&p->offsets), (size_t)(M + 1) * 4) && dalloc(&p->ws, ws_bytes) &&
       cudaMemset(p->ws, 0, ws_bytes) == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess;
  if (!ok) {
    release(p);
    return MOGA_ERR_CUDA;
  }
  *pipe = p;
  return MOGA_OK;
}

moga_status moga_pipe_submit(moga_pipe* p, const void* x, const void* W_r, const float* b_r, const void* q,
                             const void* k, const void* v, void* out, int32_t* group_id, float* gate) {
  if (!p) return MOGA_ERR_INVALID_ARG;
  if (p->N > 0 && (!x || !q || !k || !v || !out)) return MOGA_ERR_INVALID_ARG;
  if (!W_r) return MOGA_ERR_INVALID_ARG;
  DeviceScope scope(p->dev);
  if (!scope.ok) return MOGA_ERR_CUDA;
  moga_pipe::Slot& s = p->slot[p->steps & 1];
  auto fail = [p](moga_status st) {
    if (p->err == MOGA_OK) p->err = st;
    return st;
  };
  auto h2d = [p](void* dst, const void* src, size_t n) {
    return n == 0 || cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, p->s_in) == cudaSuccess;
  };
  auto d2h = [p](void* dst, const void* src, size_t n) {
    return n == 0 || cudaMemcpyAsync(dst, src, n, cudaMemcpyDeviceToHost, p->s_out) == cudaSuccess;
  };
  // copy in: the slot's inputs are free once the step two back has computed
  bool ok = !s.used || cudaStreamWaitEvent(p->s_in, s.comp_done, 0) == cudaSuccess;
  ok = ok && h2d(s.x, x, p->x_bytes) && h2d(s.w, W_r, p->w_bytes) && (!b_r || h2d(s.b, b_r, p->b_bytes)) &&
       h2d(s.q, q, p->qkv_bytes) && h2d(s.k, k, p->qkv_bytes) && h2d(s.v, v, p->qkv_bytes) &&
       cudaEventRecord(s.in_done, p->s_in) == cudaSuccess;
  // compute: after the inputs arrived and the step two back copied its output out
  ok = ok && cudaStreamWaitEvent(p->s_comp, s.in_done, 0) == cudaSuccess &&
       (!s.used || cudaStreamWaitEvent(p->s_comp, s.out_done, 0) == cudaSuccess);
  if (!ok) return fail(MOGA_ERR_CUDA);
  const moga_status st =
      moga_layer_ex(s.x, s.w, b_r ? s.b : nullptr, p->x_dt, s.q, s.k, s.v, p->N, p->d, p->H, p->d_h, p->M, p->T,
                    p->Hg, p->Wg, p->has_window ? p->window : nullptr, p->branches, s.out, s.gid, s.gate, p->perm,
                    p->offsets, p->ws, p->ws_bytes, p->s_comp);
  // The events are recorded even after a failed launch, so the slot chain
  // stays consistent for later steps.
  ok = cudaEventRecord(s.comp_done, p->s_comp) == cudaSuccess;
  // copy out
  ok = ok && cudaStreamWaitEvent(p->s_out, s.comp_done, 0) == cudaSuccess && d2h(out, s.out, p->qkv_bytes) &&
       (!group_id || d2h(group_id, s.gid, p->tok_bytes)) && (!gate || d2h(gate, s.gate, p->tok_bytes)) &&
       cudaEventRecord(s.out_done, p->s_out) == cudaSuccess;
  s.used = true;
  ++p->steps;
  if (st != MOGA_OK) return fail(st);
  if (!ok) return fail(MOGA_ERR_CUDA);
  return MOGA_OK;
}

moga_status moga_pipe_sync(moga_pipe* p) {
  if (!p) return MOGA_ERR_INVALID_ARG;
  DeviceScope scope(p->dev);
  if (!scope.ok) return MOGA_ERR_CUDA;
  bool ok = cudaStreamSynchronize(p->s_in) == cudaSuccess;
  ok = cudaStreamSynchronize(p->s_out) == cudaSuccess && ok;  // waits for compute too (event chain)
  const moga_status dev = moga_sync_status(p->ws, p->s_comp);
  moga_status st = p->err;
  p->err = MOGA_OK;
  if (st == MOGA_OK && !ok) st = MOGA_ERR_CUDA;
  if (st == MOGA_OK) st = dev;
  return st;
}

moga_status moga_pipe_destroy(moga_pipe* p) {
  if (!p) return MOGA_OK;
  DeviceScope scope(p->dev);
  release(p);
  return MOGA_OK;
}

}  // extern "C"
