// Shot-aware STGA windows ("MoGA: Mixture-of-Groups Attention for End-to-End
// Long Video Generation", §3.4 "Spatial-Temporal Group Attention (STGA)"):
// temporal groups never cross a shot cut, and the keys and values (not the
// queries) of a shot's boundary windows are augmented with latent frames of
// the adjacent shots.
//
// shot_table_kernel  one CTA: checks the shot boundaries, enumerates the
//                    windows (shot, temporal window, tile row, tile column),
//                    and scans their query / key-value lengths and work units
//                    into the window table (layout in internal.h).
// shot_perm_kernel   query index list (every token once, window by window)
//                    and key/value index list (each window's own tokens, then
//                    its previous-shot frames, then its next-shot frames).
#include <cuda_runtime.h>

#include "internal.h"

namespace moga {

namespace {

constexpr int kScanThreads = 1024;

// Exclusive prefix of v over the 1024 threads of the block; *total receives
// the block sum.  Every thread of the block must call it.
__device__ int block_excl_scan(int v, int* total) {
  __shared__ int warp_sums[32];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int s = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    warp_sums[lane] = s;
  }
  __syncthreads();
  const int before = wid ? warp_sums[wid - 1] : 0;
  *total = warp_sums[31];
  __syncthreads();
  return before + x - v;
}

__global__ void __launch_bounds__(kScanThreads)
shot_table_kernel(const int32_t* __restrict__ ss, int S, int T, int Hg, int Wg, int wt, int wh, int ww, int ap,
                  int an, int H, int cap, int32_t* __restrict__ wtab, int* status) {
  __shared__ int bad;
  int32_t* pre = wtab + kShotHdr;
  int32_t* ent = wtab + kShotHdr + cap + 1;
  const int tid = threadIdx.x;
  if (tid == 0) bad = 0;
  __syncthreads();
  for (int j = tid; j < S; j += kScanThreads) {
    const int a = ss[j], b = ss[j + 1];
    if (a >= b || (j == 0 && a != 0) || (j == S - 1 && b != T)) bad = 1;
  }
  __syncthreads();
  const int nwh = (Hg + wh - 1) / wh, nww = (Wg + ww - 1) / ww, tiles = nwh * nww;
  // windows of each shot -> first window of each shot (kept in pre[] for now)
  int nwin = 0;
  if (!bad) {
    for (int j0 = 0; j0 < S; j0 += kScanThreads) {
      const int j = j0 + tid;
      int cnt = 0;
      if (j < S) {
        const int len = ss[j + 1] - ss[j];
        cnt = (wt > 0 ? (len + wt - 1) / wt : 1) * tiles;
      }
      int tot = 0;
      const int ex = block_excl_scan(cnt, &tot);
      if (j < S && nwin + ex <= cap) pre[j] = nwin + ex;
      nwin += tot;
    }
  }
  if (bad || nwin > cap) {  // uniform over the block
    if (tid == 0) {
      wtab[0] = wtab[1] = wtab[2] = wtab[3] = 0;
      if (status) atomicOr(status, DEV_RANGE);
    }
    return;
  }
  __syncthreads();
  // per window: frames, tile and lengths
  for (int w = tid; w < nwin; w += kScanThreads) {
    int lo = 0, hi = S - 1;  // the shot of window w: largest j with pre[j] <= w
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pre[mid] <= w) lo = mid; else hi = mid - 1;
    }
    const int j = lo, local = w - pre[j];
    const int ti = local / tiles, tile = local - ti * tiles;
    const int th = tile / nww, tc = tile - th * nww;
    const int a = ss[j], b = ss[j + 1];
    const int step = wt > 0 ? wt : b - a;
    const int t0 = a + ti * step, t1 = min(b, t0 + step);
    int pf0 = 0, pf1 = 0, nf0 = 0, nf1 = 0;
    if (t0 == a && j > 0) {
      pf0 = max(ss[j - 1], a - ap);
      pf1 = a;
    }
    if (t1 == b && j < S - 1) {
      nf0 = b;
      nf1 = min(ss[j + 2], b + an);
    }
    const int area = (min(Hg, th * wh + wh) - th * wh) * (min(Wg, tc * ww + ww) - tc * ww);
    int32_t* e = ent + (size_t)w * kShotEnt;
    e[1] = (t1 - t0) * area;
    e[3] = (t1 - t0 + pf1 - pf0 + nf1 - nf0) * area;
    e[4] = t0;
    e[5] = t1;
    e[6] = pf0;
    e[7] = pf1;
    e[8] = nf0;
    e[9] = nf1;
    e[10] = th;
    e[11] = tc;
  }
  __syncthreads();
  // segment starts and the work-unit prefix (query-tile pairs x heads)
  int cq = 0, ckv = 0, cu = 0;
  for (int w0 = 0; w0 < nwin; w0 += kScanThreads) {
    const int w = w0 + tid;
    int ql = 0, kl = 0, un = 0;
    if (w < nwin) {
      const int32_t* e = ent + (size_t)w * kShotEnt;
      ql = e[1];
      kl = e[3];
      un = (((ql + kTile - 1) / kTile + 1) / 2) * H;
    }
    int tq = 0, tk = 0, tu = 0;
    const int xq = block_excl_scan(ql, &tq);
    const int xk = block_excl_scan(kl, &tk);
    const int xu = block_excl_scan(un, &tu);
    if (w < nwin) {
      int32_t* e = ent + (size_t)w * kShotEnt;
      e[0] = cq + xq;
      e[2] = ckv + xk;
      pre[w] = cu + xu;
    }
    cq += tq;
    ckv += tk;
    cu += tu;
  }
  if (tid == 0) {
    pre[nwin] = cu;
    wtab[0] = nwin;
    wtab[1] = cu;
    wtab[2] = ckv;
    wtab[3] = 0;
  }
}

__global__ void __launch_bounds__(256)
shot_perm_kernel(const int32_t* __restrict__ wtab, int cap, int Hg, int Wg, int wh, int ww,
                 int32_t* __restrict__ qperm, int32_t* __restrict__ kvperm) {
  const int nwin = wtab[0];
  const int32_t* ent = wtab + kShotHdr + cap + 1;
  for (int w = blockIdx.x; w < nwin; w += gridDim.x) {
    const int32_t* e = ent + (size_t)w * kShotEnt;
    const int qs = e[0], ql = e[1], ks = e[2];
    const int t0 = e[4], pf0 = e[6], pf1 = e[7], nf0 = e[8], nf1 = e[9];
    const int h0 = e[10] * wh, w0 = e[11] * ww;
    const int cols = min(Wg, w0 + ww) - w0;
    const int area = (min(Hg, h0 + wh) - h0) * cols;
    const int np = (pf1 - pf0) * area, nn = (nf1 - nf0) * area;
    for (int i = threadIdx.x; i < ql + np + nn; i += blockDim.x) {
      int ii = i, tb = t0;
      if (i >= ql + np) {
        ii = i - ql - np;
        tb = nf0;
      } else if (i >= ql) {
        ii = i - ql;
        tb = pf0;
      }
      const int f = ii / area, rem = ii - f * area;
      const int r = rem / cols, c = rem - r * cols;
      const int tok = ((tb + f) * Hg + h0 + r) * Wg + w0 + c;
      if (i < ql) qperm[qs + i] = tok;
      kvperm[ks + i] = tok;
    }
  }
}

}  // namespace

cudaError_t launch_shot_table(const DevCtx& c, const int32_t* shot_start, int nshots, int T, int Hg, int Wg,
                              const int* window, int aug_prev, int aug_next, int H, int64_t cap, int32_t* wtab) {
  shot_table_kernel<<<1, kScanThreads, 0, c.stream>>>(shot_start, nshots, T, Hg, Wg, window[0], window[1],
                                                     window[2], aug_prev, aug_next, H, (int)cap, wtab, c.status);
  return cudaGetLastError();
}

cudaError_t launch_shot_perm(const DevCtx& c, const int32_t* wtab, int64_t cap, int Hg, int Wg, const int* window,
                             int32_t* qperm, int32_t* kvperm) {
  int64_t blocks = cap < (int64_t)c.num_sms * 8 ? cap : (int64_t)c.num_sms * 8;
  if (blocks < 1) blocks = 1;
  shot_perm_kernel<<<(unsigned)blocks, 256, 0, c.stream>>>(wtab, (int)cap, Hg, Wg, window[1], window[2], qperm,
                                                          kvperm);
  return cudaGetLastError();
}

}  // namespace moga
