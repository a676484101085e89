// Grouped attention (Algorithm 1 steps 2-4 and Eq. 5 of "MoGA: Mixture-of-
// Groups Attention for End-to-End Long Video Generation", §3.4 "Grouped
// Attention" / "MoGA Pseudocode and Kernel Integration") and STGA window
// attention (same page, "Spatial-Temporal Group Attention").
//
// gather_kernel     Q^,K^,V^[h][j] = q,k,v[perm[j]][h]: 16-byte vector copies,
//                   one warp per token row, head-major destination so that each
//                   (segment, head) is a dense [rows x d_h] matrix for TMA.
// window_perm_kernel  position of every grid token in window order (STGA).
// seg_table_kernel  groups sorted by size (largest first) with the prefix of
//                   their query-tile counts: the persistent attention grid walks
//                   this longest-first order.
// attn_kernel<DH>   persistent varlen flash attention on tcgen05.  Per CTA:
//                   warp 0 issues TMA loads (Q tile, double-buffered K/V),
//                   warp 1 issues tcgen05.mma (S = Q K^T into one of two TMEM
//                   S buffers, O += P V into a TMEM O buffer), warps 2-5 run the
//                   online softmax on one query row per thread (S read from
//                   TMEM, P written as bf16 into a 128B-swizzled smem tile, O
//                   rescaled in TMEM only when a row max grows by more than
//                   2^8), and the epilogue scales by gate/l and scatters each
//                   row to out[perm[j]] (or adds into it for the STGA branch).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace moga {

namespace {

constexpr int kAttnThreads = 192;
constexpr int kStages = 2;

__device__ __forceinline__ uint4 ldg_stream(const uint4* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

__global__ void __launch_bounds__(256)
gather_kernel(const uint4* __restrict__ q, const uint4* __restrict__ k, const uint4* __restrict__ v,
              const int32_t* __restrict__ perm, int64_t N, int H, int vph, uint4* __restrict__ qh,
              uint4* __restrict__ kh, uint4* __restrict__ vh, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int vpr = H * vph;
  for (int64_t j = w0; j < N; j += nw) {
    const int64_t src = perm[j];
    if (src < 0 || src >= N) {
      if (lane == 0 && status) atomicOr(status, DEV_RANGE);
      continue;
    }
    const uint4* qs = q + src * vpr;
    const uint4* ks = k + src * vpr;
    const uint4* vs = v + src * vpr;
#pragma unroll 2
    for (int u = lane; u < vpr; u += 32) {
      const int h = u / vph, c = u - h * vph;
      const int64_t dst = ((int64_t)h * N + j) * vph + c;
      const uint4 a = ldg_stream(qs + u);
      const uint4 b = ldg_stream(ks + u);
      const uint4 e = ldg_stream(vs + u);
      qh[dst] = a;
      kh[dst] = b;
      vh[dst] = e;
    }
  }
}

struct WinGeom {
  int T, Hg, Wg, wt, wh, ww, nbh, nbw;
};

__device__ __forceinline__ void window_of(const WinGeom& g, int seg, int& start, int& len) {
  const int tb = seg / (g.nbh * g.nbw);
  const int hb = (seg / g.nbw) % g.nbh;
  const int wb = seg % g.nbw;
  const int t0 = tb * g.wt, h0 = hb * g.wh, w0 = wb * g.ww;
  const int et = min(g.wt, g.T - t0), eh = min(g.wh, g.Hg - h0), ew = min(g.ww, g.Wg - w0);
  start = t0 * g.Hg * g.Wg + et * (h0 * g.Wg + eh * w0);
  len = et * eh * ew;
}

__global__ void window_perm_kernel(WinGeom g, int N, int32_t* __restrict__ perm_w) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  const int t = i / (g.Hg * g.Wg);
  const int h = (i / g.Wg) % g.Hg;
  const int w = i % g.Wg;
  const int tb = t / g.wt, hb = h / g.wh, wb = w / g.ww;
  const int seg = (tb * g.nbh + hb) * g.nbw + wb;
  int start, len;
  window_of(g, seg, start, len);
  const int t0 = tb * g.wt, h0 = hb * g.wh, w0 = wb * g.ww;
  const int eh = min(g.wh, g.Hg - h0), ew = min(g.ww, g.Wg - w0);
  perm_w[start + ((t - t0) * eh + (h - h0)) * ew + (w - w0)] = i;
}

// table = [tile_prefix (M+1) | seg_start (M) | seg_len (M)], groups in
// descending size order (ties: lower group first).
__global__ void __launch_bounds__(1024)
seg_table_kernel(const int32_t* __restrict__ offsets, int M, int H, int64_t N, int32_t* __restrict__ table,
                 int* status) {
  __shared__ int n_s[1024];
  __shared__ int order[1024];
  __shared__ int bad;
  const int tid = threadIdx.x;
  if (tid == 0) bad = (offsets[0] != 0 || (int64_t)offsets[M] != N) ? 1 : 0;
  if (tid < M) {
    const int n = offsets[tid + 1] - offsets[tid];
    n_s[tid] = n;
  }
  __syncthreads();
  if (tid < M && n_s[tid] < 0) bad = 1;
  __syncthreads();
  if (bad) {
    if (tid == 0) {
      if (status) atomicOr(status, DEV_RANGE);
      table[M] = 0;
      for (int r = 0; r < M; ++r) table[r] = 0;
    }
    return;
  }
  if (tid < M) {
    const int n = n_s[tid];
    int rank = 0;
    for (int g = 0; g < M; ++g) {
      const int m = n_s[g];
      rank += (m > n) || (m == n && g < tid);
    }
    order[rank] = tid;
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int r = 0; r < M; ++r) {
      const int g = order[r];
      const int n = n_s[g];
      table[r] = run;
      table[M + 1 + r] = offsets[g];
      table[2 * M + 1 + r] = n;
      run += ((n + kTile - 1) / kTile) * H;
    }
    table[M] = run;
  }
}

template <int DH>
struct Plan {
  static constexpr int kChunks = DH / 64;
  static constexpr int kTileBytes = kTile * DH * 2;  // one 128-row bf16 operand
  static constexpr int kQ = 0;
  static constexpr int kK0 = kTileBytes;
  static constexpr int kStageBytes = 2 * kTileBytes;  // K then V
  static constexpr int kP = kK0 + kStages * kStageBytes;
  static constexpr int kPBytes = kTile * kTile * 2;
  static constexpr int kBar = kP + kPBytes;
  static constexpr int kTable = kBar + 256;
  static size_t bytes(int table_ints) { return (size_t)kTable + (size_t)table_ints * 4 + 1024; }
};

struct TileInfo {
  int h, start, len, q0;
};

struct Decoder {
  const AttnArgs* a;
  const int* tab;  // shared copy of the segment table (groups)
  WinGeom g;
  int tpw;         // query tiles per window (windows)
  __device__ __forceinline__ TileInfo operator()(int idx) const {
    TileInfo t;
    if (a->mode == 0) {
      const int M = a->nseg;
      int lo = 0, hi = M - 1;  // largest r with prefix[r] <= idx
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab[mid] <= idx) lo = mid; else hi = mid - 1;
      }
      const int local = idx - tab[lo];
      t.start = tab[M + 1 + lo];
      t.len = tab[2 * M + 1 + lo];
      const int ntq = (t.len + kTile - 1) / kTile;
      t.h = local / ntq;
      t.q0 = (local - t.h * ntq) * kTile;
    } else {
      const int qt = idx % tpw;
      const int rest = idx / tpw;
      const int seg = rest % a->nseg;
      t.h = rest / a->nseg;
      window_of(g, seg, t.start, t.len);
      t.q0 = qt * kTile;
    }
    return t;
  }
};

template <int DH>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const AttnArgs a, int* status, unsigned long long wait_ns) {
  using P = Plan<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;
  uint64_t* kv_full = bars + 2;    // [kStages]
  uint64_t* kv_empty = bars + 4;   // [kStages]
  uint64_t* s_full = bars + 6;     // [2]
  uint64_t* s_empty = bars + 8;    // [2]
  uint64_t* p_full = bars + 10;
  uint64_t* o_ready = bars + 11;
  uint64_t* done_bar = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 14);
  int* tab = reinterpret_cast<int*>(smem + P::kTable);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&kv_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_ready, 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  int total;
  Decoder dec;
  dec.a = &a;
  dec.tab = tab;
  if (a.mode == 0) {
    const int n = 3 * a.nseg + 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) tab[i] = a.table[i];
  } else {
    dec.g = WinGeom{a.T, a.Hg, a.Wg, a.wt, a.wh, a.ww, (a.Hg + a.wh - 1) / a.wh, (a.Wg + a.ww - 1) / a.ww};
    dec.tpw = (a.wt * a.wh * a.ww + kTile - 1) / kTile;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  total = (a.mode == 0) ? tab[a.nseg] : a.nseg * dec.tpw * a.H;
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem;             // S buffers: columns [0,128) and [128,256)
  const uint32_t tO = tmem + 256;       // O: columns [256, 256 + DH)
  WaitCtx wc{abort_flag, status, wait_ns};
  const int64_t N = a.N;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      uint32_t it = 0, tcnt = 0;
      bool ok = true;
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        const TileInfo ti = dec(idx);
        if (ti.q0 >= ti.len) continue;
        const int nkv = (ti.len + kTile - 1) / kTile;
        if (!mbar_wait(q_empty, (tcnt & 1) ^ 1, wc)) break;
        const int rowq = (int)((int64_t)ti.h * N + ti.start + ti.q0);
        mbar_expect_tx(q_full, P::kTileBytes);
#pragma unroll
        for (int c = 0; c < P::kChunks; ++c) tma_load_2d(&tq, q_full, smem + P::kQ + c * 16384, c * 64, rowq);
        for (int kv = 0; kv < nkv; ++kv, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&kv_empty[st], ((it / kStages) & 1) ^ 1, wc)) { ok = false; break; }
          const int rowk = (int)((int64_t)ti.h * N + ti.start + kv * kTile);
          uint8_t* ks = smem + P::kK0 + st * P::kStageBytes;
          mbar_expect_tx(&kv_full[st], 2 * P::kTileBytes);
#pragma unroll
          for (int c = 0; c < P::kChunks; ++c) {
            tma_load_2d(&tk, &kv_full[st], ks + c * 16384, c * 64, rowk);
            tma_load_2d(&tv, &kv_full[st], ks + P::kTileBytes + c * 16384, c * 64, rowk);
          }
        }
        ++tcnt;
      }
      // Drain every load this thread issued before the CTA exits.
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      if (tcnt > 0) mbar_wait(q_full, (tcnt - 1) & 1, dc);
      for (int s = 0; s < kStages && (uint32_t)s < it; ++s) {
        const uint32_t last = it - 1 - ((it - 1 - s) % kStages);
        mbar_wait(&kv_full[s], (last / kStages) & 1, dc);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16(128, DH, false, true);
      const uint32_t q_addr = smem_u32(smem + P::kQ);
      const uint32_t p_addr = smem_u32(smem + P::kP);
      uint32_t it = 0, tcnt = 0, pcnt = 0;
      bool ok = true;
      auto issue_pv = [&](int st, bool acc) {
        const uint32_t v_addr = smem_u32(smem + P::kK0 + st * P::kStageBytes + P::kTileBytes);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(p_addr + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(v_addr + kk * 2048, 16384, 1024);
          umma_bf16(tO, ad, bd, idO, (acc || kk > 0) ? 1u : 0u);
        }
      };
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        const TileInfo ti = dec(idx);
        if (ti.q0 >= ti.len) continue;
        const int nkv = (ti.len + kTile - 1) / kTile;
        if (!mbar_wait(q_full, tcnt & 1, wc)) break;
        tc_fence_after();
        int prev_st = -1;
        for (int kv = 0; kv < nkv; ++kv, ++it) {
          const int st = it % kStages;
          if (!mbar_wait(&kv_full[st], (it / kStages) & 1, wc)) { ok = false; break; }
          const int sb = it & 1;
          if (!mbar_wait(&s_empty[sb], ((it >> 1) & 1) ^ 1, wc)) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + P::kK0 + st * P::kStageBytes);
#pragma unroll
          for (int kk = 0; kk < DH / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            umma_bf16(tS + sb * 128, sdesc_sw128(q_addr + off, 16, 1024), sdesc_sw128(k_addr + off, 16, 1024), idS,
                      kk > 0 ? 1u : 0u);
          }
          umma_commit(&s_full[sb]);
          if (kv == nkv - 1) umma_commit(q_empty);
          if (prev_st >= 0) {
            if (!mbar_wait(p_full, pcnt & 1, wc)) { ok = false; break; }
            ++pcnt;
            tc_fence_after();
            issue_pv(prev_st, kv - 1 > 0);
            umma_commit(&kv_empty[prev_st]);
            umma_commit(o_ready);
          }
          prev_st = st;
        }
        if (!ok) break;
        if (!mbar_wait(p_full, pcnt & 1, wc)) break;
        ++pcnt;
        tc_fence_after();
        issue_pv(prev_st, nkv - 1 > 0);
        umma_commit(&kv_empty[prev_st]);
        umma_commit(o_ready);
        ++tcnt;
      }
      umma_commit(done_bar);
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      mbar_wait(done_bar, 0, dc);
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const int sub = warp & 3;
    const int row = sub * 32 + lane;
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)DH);
    uint8_t* p_row = smem + P::kP + row * 128;
    uint32_t it = 0, ocnt = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
      const TileInfo ti = dec(idx);
      if (ti.q0 >= ti.len) continue;
      const int nkv = (ti.len + kTile - 1) / kTile;
      float m_run = -INFINITY, l = 0.f;
      for (int kv = 0; kv < nkv; ++kv, ++it) {
        const int sb = it & 1;
        if (!mbar_wait(&s_full[sb], (it >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        float s[kTile];
#pragma unroll
        for (int c = 0; c < kTile / 32; ++c) tmem_ld32(tS + lane_base + sb * 128 + c * 32, s + c * 32);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_empty[sb]);
        const int valid = min(kTile, ti.len - kv * kTile);
        float rmax = -INFINITY;
#pragma unroll
        for (int j = 0; j < kTile; ++j) {
          s[j] = (j < valid) ? s[j] * scale_log2 : -INFINITY;
          rmax = fmaxf(rmax, s[j]);
        }
        if (kv > 0) {
          // O and the P buffer are busy until the previous P V product lands.
          if (!mbar_wait(o_ready, ocnt & 1, wc)) { ok = false; break; }
          ++ocnt;
          tc_fence_after();
          const bool need = rmax > m_run + 8.0f;
          if (__any_sync(0xffffffffu, need)) {
            const float alpha = need ? fast_exp2(m_run - rmax) : 1.0f;
            if (need) {
              l *= alpha;
              m_run = rmax;
            }
#pragma unroll
            for (int c = 0; c < DH / 32; ++c) {
              float o[32];
              tmem_ld32(tO + lane_base + c * 32, o);
              tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] *= alpha;
              tmem_st32(tO + lane_base + c * 32, o);
            }
            tmem_st_wait();
          }
        } else {
          m_run = rmax;
        }
#pragma unroll
        for (int u = 0; u < kTile / 8; ++u) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = fast_exp2(s[u * 8 + e] - m_run);
            l += p[e];
          }
          uint4 pk;
          pk.x = pack_bf16x2(p[0], p[1]);
          pk.y = pack_bf16x2(p[2], p[3]);
          pk.z = pack_bf16x2(p[4], p[5]);
          pk.w = pack_bf16x2(p[6], p[7]);
          *reinterpret_cast<uint4*>(p_row + (u >> 3) * 16384 + (((u & 7) ^ (row & 7)) << 4)) = pk;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok) break;
      // epilogue: wait for the last P V product, normalise, gate, scatter
      if (!mbar_wait(o_ready, ocnt & 1, wc)) break;
      ++ocnt;
      tc_fence_after();
      const int r = ti.q0 + row;
      bool live = r < ti.len;
      int64_t src = 0;
      if (live) {
        src = a.perm[ti.start + r];
        if (src < 0 || src >= N) {
          live = false;
          if (status) atomicOr(status, DEV_RANGE);
        }
      }
      const float gt = (live && a.gate) ? a.gate[src] : 1.0f;
      const float inv = a.out_scale * gt / l;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + (src * a.H + ti.h) * (int64_t)DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        float o[32];
        tmem_ld32(tO + lane_base + c * 32, o);
        tmem_ld_wait();
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = o[u * 8 + e] * inv;
            if (a.accumulate) {
              const uint4 old = dst[u];
              const __nv_bfloat162* ob = reinterpret_cast<const __nv_bfloat162*>(&old);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(ob[e]);
                w[2 * e] += f.x;
                w[2 * e + 1] += f.y;
              }
            }
            uint4 pk;
            pk.x = pack_bf16x2(w[0], w[1]);
            pk.y = pack_bf16x2(w[2], w[3]);
            pk.z = pack_bf16x2(w[4], w[5]);
            pk.w = pack_bf16x2(w[6], w[7]);
            dst[u] = pk;
          }
        }
      }
      tc_fence_before();
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DH>
cudaError_t launch_attention_dh(const DevCtx& c, const AttnArgs& a) {
  using P = Plan<DH>;
  CUtensorMap mq, mk, mv;
  const uint64_t rows = (uint64_t)a.N * (uint64_t)a.H;
  if (!make_tmap_2d(&mq, a.qh, DH, rows, DH * 2, kTile)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&mk, a.kh, DH, rows, DH * 2, kTile)) return cudaErrorInvalidValue;
  if (!make_tmap_2d(&mv, a.vh, DH, rows, DH * 2, kTile)) return cudaErrorInvalidValue;
  const int table_ints = a.mode == 0 ? 3 * a.nseg + 1 : 0;
  const size_t smem = P::bytes(table_ints);
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = c.num_sms;
  if (a.mode == 1) {
    const int64_t tpw = ceil_div((int64_t)a.wt * a.wh * a.ww, kTile);
    const int64_t total = (int64_t)a.nseg * tpw * a.H;
    if (total < grid) grid = (int)total;
  }
  if (grid < 1) return cudaSuccess;
  attn_kernel<DH><<<grid, kAttnThreads, smem, c.stream>>>(mq, mk, mv, a, c.status, (unsigned long long)c.wait_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gather(const DevCtx& c, const void* q, const void* k, const void* v, const int32_t* perm,
                          int64_t N, int H, int d_h, void* qh, void* kh, void* vh) {
  if (N == 0) return cudaSuccess;
  const int vph = d_h / 8;
  int64_t blocks = ceil_div(N, 8);
  const int64_t cap = (int64_t)c.num_sms * 8;
  if (blocks > cap) blocks = cap;
  gather_kernel<<<(unsigned)blocks, 256, 0, c.stream>>>((const uint4*)q, (const uint4*)k, (const uint4*)v, perm, N,
                                                         H, vph, (uint4*)qh, (uint4*)kh, (uint4*)vh, c.status);
  return cudaGetLastError();
}

cudaError_t launch_window_perm(const DevCtx& c, int T, int Hg, int Wg, const int* w, int32_t* perm_w) {
  const int N = T * Hg * Wg;
  if (N == 0) return cudaSuccess;
  WinGeom g{T, Hg, Wg, w[0], w[1], w[2], (int)ceil_div(Hg, w[1]), (int)ceil_div(Wg, w[2])};
  window_perm_kernel<<<(unsigned)ceil_div(N, 256), 256, 0, c.stream>>>(g, N, perm_w);
  return cudaGetLastError();
}

cudaError_t launch_seg_table(const DevCtx& c, const int32_t* offsets, int M, int H, int64_t N, int32_t* table) {
  seg_table_kernel<<<1, 1024, 0, c.stream>>>(offsets, M, H, N, table, c.status);
  return cudaGetLastError();
}

cudaError_t launch_attention(const DevCtx& c, const AttnArgs& a) {
  if (a.d_h == 128) return launch_attention_dh<128>(c, a);
  if (a.d_h == 64) return launch_attention_dh<64>(c, a);
  return cudaErrorInvalidValue;
}

}  // namespace moga
