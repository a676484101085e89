// Router (Eqs. 2-4 of "MoGA: Mixture-of-Groups Attention for End-to-End Long
// Video Generation", §3.4 "MoGA Router") and the index half of Algorithm 1,
// step 2 (counting sort of tokens by group).
//
// route_tc_kernel   bf16 x: persistent tcgen05 skinny GEMM.  Each CTA streams
//                   128-token x tiles and the matching W_r slices through a
//                   TMA ring; one thread issues tcgen05.mma into a double-
//                   buffered TMEM accumulator (128 lanes x M_pad columns); four
//                   epilogue warps read one token row each and fuse bias,
//                   softmax gate, first-index argmax and the tile histogram
//                   (global atomics into a zeroed [tiles][M] array).
// route_simt_kernel fp32 x (and M > 256): plain FMA dot products, same epilogue.
// scan_kernel       per-tile histograms -> per-tile group bases, offsets, max.
// scatter_kernel    stable rank of each token inside its tile (warp match +
//                   popcount) -> perm.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace moga {

namespace {

constexpr int kRouteThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2-5 epilogue
constexpr int kRouteMaxMPad = 256;

// 64-column chunks of x per ring stage: a stage loads kRouteChunks adjacent
// 128-byte pieces of each of its 128 rows back to back, so DRAM sees
// kRouteChunks * 128 contiguous bytes per row (long rows of large d models
// otherwise arrive as scattered 128-byte pieces).
#ifndef MOGA_ROUTE_CHUNKS
#define MOGA_ROUTE_CHUNKS 2
#endif
constexpr int kRouteChunks = MOGA_ROUTE_CHUNKS;

struct RouteSmemPlan {
  int mpad, stages, stage_bytes, x_bytes, w_bytes;
  size_t total;
};

inline RouteSmemPlan route_plan(int M) {
  RouteSmemPlan p;
  p.mpad = (int)align_up((size_t)M, 16);
  if (p.mpad < 16) p.mpad = 16;
  p.x_bytes = kTile * 128 * kRouteChunks;
  p.w_bytes = p.mpad * 128 * kRouteChunks;
  p.stage_bytes = p.x_bytes + p.w_bytes;
  p.stages = (int)((200 * 1024) / p.stage_bytes);
  if (p.stages > 8) p.stages = 8;
  if (p.stages < 2) p.stages = 2;
  // ring + barriers/histogram + alignment slack
  p.total = (size_t)p.stages * p.stage_bytes + 1024 + 4096 + 1024;
  return p;
}

// Online (max, argmax, sum of exp) update over logits in ascending group order.
// Strict '>' keeps the lowest index on exact ties.
__device__ __forceinline__ void online_softmax_step(float r, int j, float& mx, int& arg, float& sum) {
  if (r > mx) {
    sum = sum * expf(mx - r) + 1.0f;
    mx = r;
    arg = j;
  } else {
    sum += expf(r - mx);
  }
}

__global__ void __launch_bounds__(kRouteThreads, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
                const float* __restrict__ bias, int N, int d, int M, int mpad, int stages, int stage_bytes,
                int32_t* __restrict__ group_id, float* __restrict__ gate, int32_t* __restrict__ hist,
                float* __restrict__ pstat, float* __restrict__ logits, int* status, unsigned long long wait_ns) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint8_t* ring = smem;
  uint8_t* tail = ring + (size_t)stages * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(tail);
  uint64_t* empty = full + 8;
  uint64_t* acc_full = empty + 8;
  uint64_t* acc_empty = acc_full + 2;
  uint64_t* done_bar = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = (N + kTile - 1) / kTile;
  const int nk = (d + 64 * kRouteChunks - 1) / (64 * kRouteChunks);  // ring stages per tile
  const uint32_t x_bytes = kTile * 128 * kRouteChunks, w_bytes = (uint32_t)mpad * 128 * kRouteChunks;
  uint32_t ncols = 32;
  while (ncols < (uint32_t)(2 * mpad)) ncols <<= 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  WaitCtx wc{abort_flag, status, wait_ns};

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmap_x);
      tma_prefetch_desc(&tmap_w);
      uint32_t it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % stages;
          if (!mbar_wait(&empty[s], ((it / stages) & 1) ^ 1, wc)) { ok = false; break; }
          uint8_t* xs = ring + (size_t)s * stage_bytes;
          mbar_expect_tx(&full[s], x_bytes + w_bytes);  // boxes past d are zero-filled, still full size
#pragma unroll
          for (int c = 0; c < kRouteChunks; ++c)
            tma_load_2d(&tmap_x, &full[s], xs + c * (kTile * 128), (kc * kRouteChunks + c) * 64, t * kTile);
#pragma unroll
          for (int c = 0; c < kRouteChunks; ++c)
            tma_load_2d(&tmap_w, &full[s], xs + x_bytes + c * (mpad * 128), (kc * kRouteChunks + c) * 64, 0);
        }
      }
      // Drain: every issued load must land before the CTA may exit.
      const uint32_t issued = it;
      for (int s = 0; s < stages && (uint32_t)s < issued; ++s) {
        const uint32_t last = issued - 1 - ((issued - 1 - s) % stages);
        WaitCtx dc{abort_flag, nullptr, 100000000ull};
        volatile int zero = 0;
        dc.abort_flag = &zero;
        mbar_wait(&full[s], (last / stages) & 1, dc);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, mpad, false, false);
      uint32_t it = 0, tc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tc) {
        const int ab = tc & 1;
        if (!mbar_wait(&acc_empty[ab], ((tc >> 1) & 1) ^ 1, wc)) break;
        tc_fence_after();
        const uint32_t dt = tmem + (uint32_t)(ab * mpad);
        for (int kc = 0; kc < nk; ++kc, ++it) {
          const int s = it % stages;
          if (!mbar_wait(&full[s], (it / stages) & 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t xa = smem_u32(ring + (size_t)s * stage_bytes);
          const uint32_t wa = xa + x_bytes;
          const uint64_t xd = sdesc_sw128(xa, 16, 1024), wd = sdesc_sw128(wa, 16, 1024);
#pragma unroll
          for (int c = 0; c < kRouteChunks; ++c) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16(dt, sdesc_add(xd, c * (kTile * 128) + kk * 32), sdesc_add(wd, c * (mpad * 128) + kk * 32),
                        idesc, (kc | c | kk) != 0);
          }
          umma_commit(&empty[s]);
        }
        if (!ok) break;
        umma_commit(&acc_full[ab]);
      }
      // All MMAs issued by this thread must finish before TMEM is released.
      umma_commit(done_bar);
      WaitCtx dc{abort_flag, nullptr, 100000000ull};
      volatile int zero = 0;
      dc.abort_flag = &zero;
      mbar_wait(done_bar, 0, dc);
    }
  } else {
    // Epilogue: warps 2..5 -> TMEM sub-partitions 2,3,0,1.
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    uint32_t tc = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++tc) {
      const int ab = tc & 1;
      if (!mbar_wait(&acc_full[ab], (tc >> 1) & 1, wc)) break;
      tc_fence_after();
      const uint32_t base = tmem + ((uint32_t)(sub * 32) << 16) + (uint32_t)(ab * mpad);
      float mx = -INFINITY, sum = 0.f;
      int arg = 0;
      for (int c0 = 0; c0 < mpad; c0 += 16) {
        float v[16];
        tmem_ld16(base + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int col = c0 + j;
          if (col < M) online_softmax_step(v[j] + (bias ? __ldg(bias + col) : 0.f), col, mx, arg, sum);
        }
        if (logits && (int64_t)t * kTile + row < N) {
          float* lr = logits + ((int64_t)t * kTile + row) * M + c0;
          float o[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) o[j] = v[j] + ((bias && c0 + j < M) ? __ldg(bias + c0 + j) : 0.f);
          if ((M & 3) == 0 && c0 + 16 <= M) {  // rows start 16-byte aligned
#pragma unroll
            for (int q = 0; q < 4; ++q)
              reinterpret_cast<float4*>(lr)[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (c0 + j < M) lr[j] = o[j];
          }
        }
      }
      const int64_t tok = (int64_t)t * kTile + row;
      if (pstat) {
        // Balancing statistics: this warp's sum over its 32 tokens of
        // p(i|x) for every group i (butterfly reduction, fixed order).
        const float inv = 1.0f / sum;
        for (int c0 = 0; c0 < mpad; c0 += 16) {
          float v[16];
          tmem_ld16(base + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int col = c0 + j;
            float pj = (col < M && tok < N) ? expf(v[j] + (bias ? __ldg(bias + col) : 0.f) - mx) * inv : 0.f;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) pj += __shfl_xor_sync(0xffffffffu, pj, o);
            if (lane == 0 && col < M) pstat[((int64_t)t * 4 + sub) * M + col] = pj;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[ab]);
      if (tok < N) {
        group_id[tok] = arg;
        gate[tok] = 1.0f / sum;
        atomicAdd(&hist[(int64_t)t * M + arg], 1);  // hist is zeroed by the launcher
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, ncols);
  }
}

// SIMT router: one warp per token, fp32 accumulation.  Used for fp32 inputs
// and for M beyond the tensor-core path's 256 columns.
template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T>
__global__ void __launch_bounds__(128)
route_simt_kernel(const T* __restrict__ x, const T* __restrict__ W, const float* __restrict__ bias, int N, int d,
                  int M, int32_t* __restrict__ group_id, float* __restrict__ gate, int32_t* __restrict__ hist,
                  float* __restrict__ pstat, float* __restrict__ logits) {
  extern __shared__ float logit_s[];          // [4][M]
  int* hist_s = reinterpret_cast<int*>(logit_s + 4 * M);  // [M]
  float* ps = logit_s + 5 * M;                           // [4][M] per-warp sums of p(i|x)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x;
  for (int m = threadIdx.x; m < M; m += blockDim.x) hist_s[m] = 0;
  for (int m = threadIdx.x; m < 4 * M; m += blockDim.x) ps[m] = 0.f;
  __syncthreads();
  float* lg = logit_s + warp * M;
  for (int r = warp; r < kTile; r += 4) {
    const int64_t tok = (int64_t)t * kTile + r;
    if (tok >= N) break;
    const T* xr = x + tok * d;
    for (int m = 0; m < M; ++m) {
      const T* wr = W + (int64_t)m * d;
      float acc = 0.f;
      for (int c = lane; c < d; c += 32) acc = fmaf(to_f(xr[c]), to_f(wr[c]), acc);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      if (lane == 0) lg[m] = acc + (bias ? bias[m] : 0.f);
    }
    __syncwarp();
    if (logits)
      for (int m = lane; m < M; m += 32) logits[tok * M + m] = lg[m];
    if (lane == 0) {
      float mx = -INFINITY, sum = 0.f;
      int arg = 0;
      for (int m = 0; m < M; ++m) online_softmax_step(lg[m], m, mx, arg, sum);
      group_id[tok] = arg;
      gate[tok] = 1.0f / sum;
      atomicAdd(&hist_s[arg], 1);
      if (pstat)
        for (int m = 0; m < M; ++m) ps[warp * M + m] += expf(lg[m] - mx) / sum;
    }
    __syncwarp();
  }
  __syncthreads();
  for (int m = threadIdx.x; m < M; m += blockDim.x) hist[(int64_t)t * M + m] = hist_s[m];
  if (pstat)
    for (int m = threadIdx.x; m < 4 * M; m += blockDim.x) pstat[(int64_t)t * 4 * M + m] = ps[m];
}

// One CTA: column sums of hist per group in C chunks, exclusive scans, bases.
__global__ void __launch_bounds__(1024)
scan_kernel(const int32_t* __restrict__ hist, int ntiles, int M, int32_t* __restrict__ base,
            int32_t* __restrict__ offsets, int32_t* __restrict__ max_seqlen, const float* __restrict__ pstat,
            int N, float* __restrict__ prob_mean, float* __restrict__ balance) {
  __shared__ int part[1024];
  __shared__ int offs_s[1025];
  __shared__ float fpart[1024];
  __shared__ float pm_s[1024];
  const int C = max(1, 1024 / M);
  const int tid = threadIdx.x;
  const int per = (ntiles + C - 1) / C;
  const bool active = tid < C * M;
  const int g = active ? tid % M : 0, c = active ? tid / M : 0;
  const int t0 = c * per, t1 = min(ntiles, t0 + per);
  if (active) {
    int s = 0;
    for (int t = t0; t < t1; ++t) s += hist[(int64_t)t * M + g];
    part[c * M + g] = s;
    if (pstat) {
      // mean routing probability: per-tile, per-warp partials summed in a
      // fixed order (tile, then warp), so the result is deterministic
      float f = 0.f;
      for (int t = t0; t < t1; ++t)
        for (int w = 0; w < 4; ++w) f += pstat[((int64_t)t * 4 + w) * M + g];
      fpart[c * M + g] = f;
    }
  }
  __syncthreads();
  if (pstat && tid < M) {
    float f = 0.f;
    for (int cc = 0; cc < C; ++cc) f += fpart[cc * M + tid];
    pm_s[tid] = f / (float)N;
    if (prob_mean) prob_mean[tid] = pm_s[tid];
  }
  if (tid < M) {
    int run = 0;
    for (int cc = 0; cc < C; ++cc) {
      const int v = part[cc * M + tid];
      part[cc * M + tid] = run;
      run += v;
    }
    offs_s[tid] = run;  // group total for now
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0, mx = 0;
    for (int m = 0; m < M; ++m) {
      const int v = offs_s[m];
      offs_s[m] = run;
      offsets[m] = run;
      run += v;
      mx = max(mx, v);
    }
    offs_s[M] = run;
    offsets[M] = run;
    *max_seqlen = mx;
    if (pstat && balance) {
      // M * sum_i F_i P_i with F_i the fraction of tokens routed to group i
      float b = 0.f;
      for (int m = 0; m < M; ++m) b += ((float)(offs_s[m + 1] - offs_s[m]) / (float)N) * pm_s[m];
      *balance = (float)M * b;
    }
  }
  __syncthreads();
  if (active) {
    int run = offs_s[g] + part[c * M + g];
    for (int t = t0; t < t1; ++t) {
      base[(int64_t)t * M + g] = run;
      run += hist[(int64_t)t * M + g];
    }
  }
}

__global__ void __launch_bounds__(128)
scatter_kernel(const int32_t* __restrict__ group_id, const int32_t* __restrict__ base, int N, int M,
               int32_t* __restrict__ perm) {
  extern __shared__ int cnt[];  // [4][M]
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < 4 * M; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  const int t = blockIdx.x;
  const int64_t tok = (int64_t)t * kTile + threadIdx.x;
  const int g0 = tok < N ? group_id[tok] : -1;
  const bool valid = g0 >= 0 && g0 < M;  // ids out of range were reported by the histogram and are skipped
  const int g = valid ? g0 : -1;
  const unsigned peers = __match_any_sync(0xffffffffu, g);
  unsigned lt;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(lt));
  const int rank = __popc(peers & lt);
  if (valid && rank == 0) cnt[warp * M + g] = __popc(peers);
  __syncthreads();
  if (valid) {
    int pre = 0;
    for (int w = 0; w < warp; ++w) pre += cnt[w * M + g];
    perm[base[(int64_t)t * M + g] + pre + rank] = (int32_t)tok;
  }
}

}  // namespace

cudaError_t launch_route_tc(const DevCtx& c, const void* x, const void* W, const float* b, int64_t N, int d,
                            int M, int32_t* group_id, float* gate, int32_t* hist, float* pstat, float* logits) {
  const RouteSmemPlan p = route_plan(M);
  if (p.mpad > kRouteMaxMPad) return cudaErrorInvalidValue;
  CUtensorMap mx, mw;
  if (!make_tmap_2d(&mx, x, (uint64_t)d, (uint64_t)N, (uint64_t)d * 2, kTile)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&mw, W, (uint64_t)d, (uint64_t)M, (uint64_t)d * 2, (uint32_t)p.mpad))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(route_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.total);
  if (e != cudaSuccess) return e;
  const int64_t ntiles = ceil_div(N, kTile);
  e = cudaMemsetAsync(hist, 0, (size_t)ntiles * M * sizeof(int32_t), c.stream);
  if (e != cudaSuccess) return e;
  const int grid = (int)(ntiles < c.num_sms ? ntiles : c.num_sms);
  route_tc_kernel<<<grid, kRouteThreads, p.total, c.stream>>>(mx, mw, b, (int)N, d, M, p.mpad, p.stages,
                                                               p.stage_bytes, group_id, gate, hist, pstat, logits,
                                                               c.status,
                                                               (unsigned long long)c.wait_ns);
  return cudaGetLastError();
}

cudaError_t launch_route_simt(const DevCtx& c, const void* x, const void* W, const float* b, bool bf16,
                              int64_t N, int d, int M, int32_t* group_id, float* gate, int32_t* hist, float* pstat,
                              float* logits) {
  const int64_t ntiles = ceil_div(N, kTile);
  const size_t smem = (size_t)9 * M * sizeof(float);
  if (bf16) {
    auto k = route_simt_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<(unsigned)ntiles, 128, smem, c.stream>>>((const __nv_bfloat16*)x, (const __nv_bfloat16*)W, b, (int)N, d,
                                                  M, group_id, gate, hist, pstat, logits);
  } else {
    auto k = route_simt_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<(unsigned)ntiles, 128, smem, c.stream>>>((const float*)x, (const float*)W, b, (int)N, d, M, group_id,
                                                  gate, hist, pstat, logits);
  }
  return cudaGetLastError();
}

cudaError_t launch_scan(const DevCtx& c, const int32_t* hist, int64_t ntiles, int M, int32_t* base,
                        int32_t* offsets, int32_t* max_seqlen, const float* pstat, int64_t N, float* prob_mean,
                        float* balance) {
  scan_kernel<<<1, 1024, 0, c.stream>>>(hist, (int)ntiles, M, base, offsets, max_seqlen, pstat, (int)N, prob_mean,
                                        balance);
  return cudaGetLastError();
}

// Per-tile histograms of given group ids (moga_sort); ids outside [0, M) are
// skipped and reported.
__global__ void __launch_bounds__(128)
hist_kernel(const int32_t* __restrict__ group_id, int N, int M, int32_t* __restrict__ hist, int* status) {
  extern __shared__ int h[];  // [M]
  for (int i = threadIdx.x; i < M; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const int64_t tok = (int64_t)blockIdx.x * kTile + threadIdx.x;
  if (tok < N) {
    const int g = group_id[tok];
    if (g >= 0 && g < M)
      atomicAdd(&h[g], 1);
    else if (status)
      atomicOr(status, DEV_RANGE);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < M; i += blockDim.x) hist[(int64_t)blockIdx.x * M + i] = h[i];
}

cudaError_t launch_hist(const DevCtx& c, const int32_t* group_id, int64_t N, int M, int32_t* hist) {
  const int64_t ntiles = ceil_div(N, kTile);
  hist_kernel<<<(unsigned)ntiles, 128, (size_t)M * sizeof(int), c.stream>>>(group_id, (int)N, M, hist, c.status);
  return cudaGetLastError();
}

cudaError_t launch_scatter(const DevCtx& c, const int32_t* group_id, const int32_t* base, int64_t N, int M,
                           int32_t* perm) {
  const int64_t ntiles = ceil_div(N, kTile);
  const size_t smem = (size_t)4 * M * sizeof(int);
  scatter_kernel<<<(unsigned)ntiles, 128, smem, c.stream>>>(group_id, base, (int)N, M, perm);
  return cudaGetLastError();
}

}  // namespace moga
