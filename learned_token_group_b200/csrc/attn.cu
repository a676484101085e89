// Grouped attention (Algorithm 1 steps 2-4 and Eq. 5 of "MoGA: Mixture-of-
// Groups Attention for End-to-End Long Video Generation", §3.4 "Grouped
// Attention" / "MoGA Pseudocode and Kernel Integration") and STGA window
// attention (same page, "Spatial-Temporal Group Attention").
//
// window_perm_kernel  position of every grid token in window order (STGA).
// seg_table_kernel  groups sorted by size (largest first) with the prefix of
//                   their query-tile counts: the persistent attention grid walks
//                   this longest-first order.
// attn_kernel<DH>   persistent varlen flash attention on tcgen05.  A CTA works
//                   on two 128-row query tiles (A, B) of one (segment, head)
//                   at a time, streaming the segment's K/V tiles once for both.
//                   Loads: grouped attention (and large windows) read 128-row
//                   tiles of a gathered head-major copy with 2-D TMA (warp 0);
//                   whole-frame windows read 128 consecutive tokens in place
//                   with 3-D TMA; STGA windows of 193 to 256 tokens and short
//                   shot windows are copied straight from q, k, v by token
//                   index with cp.async by warps 0, 2 and 3.  (STGA windows of
//                   up to 192 tokens run stga_kernel, stga.cu.)
//                   Warp 1 issues tcgen05.mma in the order
//                   PV_A(j), S_A(j+1), PV_B(j), S_B(j+1), so the tensor core
//                   works on one tile while the other tile's softmax runs;
//                   warps 4-7 and 8-11 are the two softmax warpgroups (one query
//                   row per thread): S is read from TMEM, P is written back as
//                   bf16 over S in TMEM and consumed from there by the P V
//                   product, O is rescaled in TMEM only when a row max grows by
//                   more than 2^8; the epilogue scales by gate/l and scatters
//                   each row to out[perm[j]] (or, for a later branch of the
//                   block, adds into it with vector reductions).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <type_traits>

#include "internal.h"
#include "ptx.cuh"
#include "windows.cuh"

namespace moga {

namespace {

// One key pair in every kExp2PolyEvery goes through the FMA-pipe polynomial
// instead of MUFU ex2 (0 disables), balancing the two units in the softmax.
#ifndef MOGA_EXP2_POLY_EVERY
#define MOGA_EXP2_POLY_EVERY 8
#endif
constexpr int kExp2PolyEvery = MOGA_EXP2_POLY_EVERY;
// Warpgroup 0: warp 0 TMA, warp 1 MMA (+ TMEM allocation), warps 2-3 idle;
// warpgroups 1 and 2: softmax + epilogue of query tiles A and B.
constexpr int kAttnThreads = 384;
// Register split after launch (384 threads x 168): warpgroup 0 drops to 104,
// the softmax warpgroups rise to 192: 128*104 + 256*192 = 62464 <= 64512
// (multiples of 8; this split compiles without spills).
constexpr int kRegsCtl = 104;
constexpr int kRegsSoftmax = 192;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kAttnThreads * 168, "register split exceeds the launch");
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

// da[h][j] = a[idx[j]][h] (and db from b when given) for j < rows, where rows
// is *rows_dev when given (a count the device computed) else rows_max; the
// destinations are head-major with a per-head row stride.  Used for the
// query and key/value lists of shot windows, whose lengths differ.
__global__ void __launch_bounds__(256)
gather_rows_kernel(const uint4* __restrict__ a, const uint4* __restrict__ b, const int32_t* __restrict__ idx,
                   const int32_t* __restrict__ rows_dev, int64_t rows_max, int64_t N, int H, int vph,
                   int64_t stride, uint4* __restrict__ da, uint4* __restrict__ db, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int64_t rows = rows_dev ? min((int64_t)*rows_dev, rows_max) : rows_max;
  const int vpr = H * vph;
  for (int64_t j = w0; j < rows; j += nw) {
    const int64_t src = idx[j];
    if (src < 0 || src >= N) {
      if (lane == 0 && status) atomicOr(status, DEV_RANGE);
      continue;
    }
#pragma unroll 2
    for (int u = lane; u < vpr; u += 32) {
      const int h = u / vph, c = u - h * vph;
      const int64_t dst = ((int64_t)h * stride + j) * vph + c;
      da[dst] = ldg_stream(a + src * vpr + u);
      if (b) db[dst] = ldg_stream(b + src * vpr + u);
    }
  }
  // The last tile of the last segment may read up to a tile past `rows`:
  // those rows are zeroed so that every value the tensor core reads is finite.
  const int64_t tail = min(rows + kTile, rows_max);
  for (int64_t j = rows + w0; j < tail; j += nw) {
    for (int u = lane; u < vpr; u += 32) {
      const int h = u / vph, c = u - h * vph;
      const int64_t dst = ((int64_t)h * stride + j) * vph + c;
      da[dst] = make_uint4(0, 0, 0, 0);
      if (b) db[dst] = make_uint4(0, 0, 0, 0);
    }
  }
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

// table = [unit_prefix (M+1) | seg_start (M) | seg_len (M)], groups in
// descending size order (ties: lower group first); a unit is a pair of
// 128-row query tiles of one head.
__global__ void __launch_bounds__(1024)
seg_table_kernel(const int32_t* __restrict__ offsets, int M, int H, int64_t N, int tiles_per_unit,
                 int32_t* __restrict__ table, int* status) {
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
      run += (((n + kTile - 1) / kTile + tiles_per_unit - 1) / tiles_per_unit) * H;  // units per head
    }
    table[M] = run;
  }
}

template <int DH>
struct Plan {
  static constexpr int kChunks = DH / 64;
  static constexpr int kTileBytes = kTile * DH * 2;   // one 128-row bf16 operand tile
  static constexpr int kQA = 0;                        // query tile A
  static constexpr int kQB = kTileBytes;               // query tile B
  static constexpr int kK0 = 2 * kTileBytes;           // K ring [kStages]
  static constexpr int kV0 = kK0 + kStages * kTileBytes;  // V ring [kStages]
  static constexpr int kBar = kV0 + kStages * kTileBytes;
  static constexpr int kTable = kBar + 256;
  static size_t bytes(int table_ints) { return (size_t)kTable + (size_t)table_ints * 4 + 1024; }
  static constexpr int kChunkFull = kTile * 128;  // bytes of one 64-column chunk, 128 rows
};

// A work unit is a pair of consecutive 128-row query tiles (A, B) of one
// (segment, head); both stream the same K/V tiles.
struct Unit {
  int h, start, len, q0;  // query segment; q0: first row of tile A in it (tile B starts at q0 + 128)
  int kvs, kvl;           // key/value segment (the query segment except for shot windows)
  int seg;                // STGA windows: the window's index (else -1)
};

// kShots: the decoder of the in-place kernel, which also serves shot windows
// (mode 2); the tiled kernel never sees them and keeps the smaller decoder.
template <bool kShots>
struct Decoder {
  int mode;
  int nseg;
  const int* tab;  // groups: shared copy of [unit_prefix (M+1) | seg_start (M) | seg_len (M)]
  WinGeom g;
  int upw;         // windows: units per window
  int H;           // windows read in place: heads vary fastest (0: heads outermost)
  int heads;       // shot windows: number of heads (heads vary fastest)
  const int* gtab; // shot windows: window table in device memory
  int cap;         // shot windows: table capacity
  __device__ __forceinline__ Unit operator()(int idx) const {
    Unit u;
    if (mode == 0) {
      int lo = 0, hi = nseg - 1;  // largest r with prefix[r] <= idx
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab[mid] <= idx) lo = mid; else hi = mid - 1;
      }
      const int local = idx - tab[lo];
      u.start = tab[nseg + 1 + lo];
      u.len = tab[2 * nseg + 1 + lo];
      const int npair = ((u.len + kTile - 1) / kTile + 1) / 2;
      u.h = local / npair;
      u.q0 = (local - u.h * npair) * 2 * kTile;
      u.kvs = u.start;
      u.kvl = u.len;
      u.seg = -1;
    } else if (!kShots || mode == 1) {
      // Units in place go window by window with the heads innermost, so the
      // CTAs running at once read whole token rows of q, k, v (all heads)
      // close together in time.  With a gathered head-major copy each head's
      // window is contiguous already, and heads go outermost.
      const int qp = idx % upw;
      const int rest = idx / upw;
      int seg;
      if (H > 0) {
        u.h = rest % H;
        seg = rest / H;
      } else {
        seg = rest % nseg;
        u.h = rest / nseg;
      }
      window_of(g, seg, u.start, u.len);
      u.q0 = qp * 2 * kTile;
      u.kvs = u.start;
      u.kvl = u.len;
      u.seg = seg;
    } else {
      // shot windows: binary search of the unit prefix in the global table
      const int nwin = gtab[0];
      const int* pre = gtab + kShotHdr;
      int lo = 0, hi = nwin - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pre[mid] <= idx) lo = mid; else hi = mid - 1;
      }
      const int* e = gtab + kShotHdr + cap + 1 + (size_t)lo * kShotEnt;
      const int local = idx - pre[lo];
      u.start = e[0];
      u.len = e[1];
      u.kvs = e[2];
      u.kvl = e[3];
      u.h = local % heads;
      u.q0 = (local / heads) * 2 * kTile;
      u.seg = -1;
    }
    return u;
  }
};

// kDirect: copy Q/K/V rows straight from q, k, v by token index (cp.async);
// otherwise 128-row tiles of a gathered head-major copy (2-D tiled TMA).
// kShots: the unit decoder also reads shot-window tables (mode 2); the
// grouped-attention instantiation leaves it out.
template <int DH, bool kDirect, bool kShots>
__global__ void __launch_bounds__(kAttnThreads, 1)
attn_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const AttnArgs a, int* status, unsigned long long wait_ns) {
  using P = Plan<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::kBar);
  uint64_t* q_full = bars + 0;    // query tiles A, B loaded (slot 0; slot 1 spare)
  uint64_t* q_empty = bars + 2;   // query tiles free again (slot 0; slot 1 spare)
  uint64_t* k_full = bars + 4;    // [kStages]
  uint64_t* k_empty = bars + 6;   // [kStages]
  uint64_t* v_full = bars + 8;    // [kStages]
  uint64_t* v_empty = bars + 10;  // [kStages]
  uint64_t* s_full = bars + 12;   // [2]: S of tile A / B computed
  uint64_t* p_full = bars + 14;   // [2]: P of tile A / B written (O rescaled)
  uint64_t* o_full = bars + 16;   // [2]: last P V of tile A / B done
  uint64_t* done_bar = bars + 18;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 19);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 20);
  int* tab = reinterpret_cast<int*>(smem + P::kTable);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&q_full[b], 1);
      mbar_init(&q_empty[b], 1);
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 128);
      mbar_init(&o_full[x], 1);
    }
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  Decoder<kShots> dec;
  dec.mode = a.mode;
  dec.nseg = a.nseg;
  dec.tab = tab;
  dec.upw = 1;
  dec.H = (kDirect || a.contiguous) ? a.H : 0;
  dec.heads = a.H;
  dec.gtab = a.table;
  dec.cap = a.nseg;
  if (a.mode == 0) {
    const int n = 3 * a.nseg + 1;
    for (int i = threadIdx.x; i < n; i += blockDim.x) tab[i] = a.table[i];
  } else if (a.mode == 1) {
    dec.g = WinGeom{a.T, a.Hg, a.Wg, a.wt, a.wh, a.ww, (a.Hg + a.wh - 1) / a.wh, (a.Wg + a.ww - 1) / a.ww};
    dec.upw = ((a.wt * a.wh * a.ww + kTile - 1) / kTile + 1) / 2;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total = a.mode == 0 ? tab[a.nseg] : a.mode == 1 ? a.nseg * dec.upw * a.H : a.table[1];
  const uint32_t tmem = *tmem_slot;
  // TMEM columns: S/P of tile A [0,128), S/P of tile B [128,256), O of A [256,..), O of B [384,..).
  // P (bf16, two per column) overwrites the first 64 columns of its tile's S.
  auto tS = [tmem](int x) { return tmem + (uint32_t)(x * 128); };
  auto tO = [tmem](int x) { return tmem + 256u + (uint32_t)(x * 128); };
  WaitCtx wc{abort_flag, status, wait_ns};
  const int64_t N = a.N;
  const int64_t kv_rows = a.kv_rows > 0 ? a.kv_rows : N;  // per-head rows of the K/V copies

  if (warp < 4) {
  regs_dec<kRegsCtl>();
  if (!kDirect && warp == 0) {
    // ---------------------------------------------------------------- TMA producer (tiled)
    // 128-row tiles of the gathered head-major copy [H][N][d_h] (row h*N + j).
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      uint32_t ucnt = 0, kc = 0, vc = 0;
      bool ok = true;
      // One 128-row tile of head h starting at segment position pos: a row of
      // the gathered head-major copy (rows = rows per head), or, for
      // contiguous segments, 128 consecutive tokens read in place.
      // K/V tiles are read again by every query pair of their (group, head):
      // keep them in L2; query tiles are read once
      const uint64_t pol_keep = l2_policy_evict_last(), pol_once = l2_policy_evict_first();
      auto load_tile = [&](const CUtensorMap* map, uint64_t* bar, uint8_t* dst, int h, int64_t rows, int pos,
                           uint64_t pol) {
#pragma unroll
        for (int c = 0; c < P::kChunks; ++c) {
          if (a.contiguous)
            tma_load_3d(map, bar, dst + c * 16384, c * 64, h, pos);
          else
            tma_load_2d_hint(map, bar, dst + c * 16384, c * 64, (int)((int64_t)h * rows + pos), pol);
        }
      };
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        const Unit u = dec(idx);
        if (u.q0 >= u.len) continue;
        const bool hb = u.q0 + kTile < u.len;
        const int nkv = (u.kvl + kTile - 1) / kTile;
        if (!mbar_wait(q_empty, (ucnt & 1) ^ 1, wc, 1, ucnt)) break;
        mbar_expect_tx(q_full, (hb ? 2 : 1) * P::kTileBytes);
        load_tile(&tq, q_full, smem + P::kQA, u.h, N, u.start + u.q0, pol_once);
        if (hb) load_tile(&tq, q_full, smem + P::kQB, u.h, N, u.start + u.q0 + kTile, pol_once);
        ++ucnt;
        for (int j = 0; j < nkv; ++j) {
          const int posk = u.kvs + j * kTile;
          const int ks = kc % kStages;
          if (!mbar_wait(&k_empty[ks], ((kc / kStages) & 1) ^ 1, wc, 2, kc)) { ok = false; break; }
          if (a.debug_withhold_first_k && kc == 0) {
            // Test hook: this K tile never arrives, so the MMA warp's bounded
            // wait runs out and the kernel reports a timeout.  No load is in
            // flight for it, so the slot is not counted for the drain below.
            ok = false;
            break;
          }
          mbar_expect_tx(&k_full[ks], P::kTileBytes);
          load_tile(&tk, &k_full[ks], smem + P::kK0 + ks * P::kTileBytes, u.h, kv_rows, posk, pol_keep);
          ++kc;
          const int vs = vc % kStages;
          if (!mbar_wait(&v_empty[vs], ((vc / kStages) & 1) ^ 1, wc, 3, vc)) { ok = false; break; }
          mbar_expect_tx(&v_full[vs], P::kTileBytes);
          load_tile(&tv, &v_full[vs], smem + P::kV0 + vs * P::kTileBytes, u.h, kv_rows, posk, pol_keep);
          ++vc;
        }
      }
      // Drain every load this thread issued before the CTA exits.
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      if (ucnt > 0) mbar_wait(q_full, (ucnt - 1) & 1, dc);
      for (int s = 0; s < kStages; ++s) {
        if ((uint32_t)s < kc) mbar_wait(&k_full[s], ((kc - 1 - ((kc - 1 - s) % kStages)) / kStages) & 1, dc);
        if ((uint32_t)s < vc) mbar_wait(&v_full[s], ((vc - 1 - ((vc - 1 - s) % kStages)) / kStages) & 1, dc);
      }
    }
  }
  if (kDirect && warp != 1) {
    // ---------------------------------------------------------------- cp.async loaders (warps 0, 2, 3)
    // Q/K/V rows are copied straight from q, k, v [N, H, d_h] by token index
    // (perm / kvperm: segment position -> token), so no gathered copy is ever
    // written.
    // Warp 0 copies Q_A and Q_B, warp 2 the K tiles and warp 3 the V tiles:
    // each lane moves 16-byte pieces with cp.async into the 128-byte swizzled
    // layout the MMA descriptors expect, waits for its pieces, fences them for
    // the async proxy, and lane 0 then arrives on the tile's barrier.  Each
    // empty barrier thus has one waiter that follows its phases in order.
    // Three warps keep up to 128 KB in flight, which single-row TMA gathers
    // could not (their per-instruction cost capped an SM near 8 B/cycle).
    const int li = warp == 0 ? 0 : warp - 1;  // 0: Q, 1: K, 2: V
    const int32_t* kvperm = a.kvperm ? a.kvperm : a.perm;
    constexpr int kPieces = DH * 2 / 16;       // 16-byte pieces per row
    constexpr int kRowsPerOp = 32 / kPieces;   // rows one warp-wide copy covers
    const int piece = lane % kPieces, sub = lane / kPieces;
    const int pchunk = piece >> 3;  // 64-column chunk of this lane's piece
    const int pj = piece & 7;
    int* toks = tab + li * 2 * kTile;  // this loader's token rows (two tiles for Q)
    const int H = a.H;
    uint32_t ucnt = 0, t = 0;
    bool ok = true;
    // Row indices of tile rows [pos0, pos0 + 128), four per lane: token * H + h,
    // or -1 (zero-filled) for a token out of range or a row past the segment
    // end.  Read before the slot is free so that their latency overlaps the
    // wait.
    auto fetch_rows = [&](const int32_t* idx, int pos0, int seg_end, int h, int (&tr)[4]) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int pp = pos0 + 4 * lane + i;
        const int tok = idx[min(pp, seg_end - 1)];
        tr[i] = (pp < seg_end && tok >= 0 && (int64_t)tok < N) ? tok * H + h : -1;
      }
    };
    // Issues the copies of one tile whose row indices are in tr (staged in
    // tk, 128 ints); the caller waits for them.  Only the copies covering the
    // tile's first nrows rows are issued (a warp-uniform count): rows past the
    // segment end keep what the slot held, which is finite (earlier tiles or
    // the initial zeros), and belong to masked keys or dropped queries.
    // chunk: byte stride between 64-column chunks (full or compact tile).
    auto copy_tile = [&](const void* g, uint8_t* dst, const int (&tr)[4], int* tk, int nrows, int chunk) {
#pragma unroll
      for (int i = 0; i < 4; ++i) tk[4 * lane + i] = tr[i];
      __syncwarp();
      const char* gb = static_cast<const char*>(g) + piece * 16;
      const uint32_t db = smem_u32(dst) + (uint32_t)(pchunk * chunk);
      const int nops = (min(nrows, kTile) + kRowsPerOp - 1) / kRowsPerOp;  // warp-uniform
#pragma unroll 8
      for (int i = 0; i < nops; ++i) {
        const int r = i * kRowsPerOp + sub;
        const int row = tk[r];
        const char* src = row >= 0 ? gb + (int64_t)row * (DH * 2) : gb;
        cp_async16(db + r * 128 + ((pj ^ (r & 7)) << 4), src, row >= 0 ? 16 : 0);
      }
    };
    auto finish = [&]() {
      cp_async_commit_wait_all();
      fence_proxy_async_smem();
      __syncwarp();
    };
    // Lane 0 waits; the whole warp learns the outcome.
    auto warp_wait = [&](uint64_t* bar, uint32_t parity, int site, uint32_t count) {
      int w = 1;
      if (lane == 0) w = mbar_wait(bar, parity, wc, site, count);
      return __shfl_sync(0xffffffffu, w, 0) != 0;
    };
    {
      // Rows past a segment's end are never copied, so the K and V rings
      // start as zeros: every row the tensor core reads is then finite (a
      // masked key's P is 0, and 0 times a finite V row adds nothing).
      const int off = li == 1 ? P::kK0 : P::kV0;
      const int bytes = li == 0 ? 0 : kStages * P::kTileBytes;
      uint4* ring = reinterpret_cast<uint4*>(smem + off);
      for (int i = lane; i < bytes / 16; i += 32) ring[i] = make_uint4(0, 0, 0, 0);
      fence_proxy_async_smem();
      __syncwarp();
    }
    for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
      const Unit u = dec(idx);
      if (u.q0 >= u.len) continue;
      const bool hb = u.q0 + kTile < u.len;
      const int nkv = (u.kvl + kTile - 1) / kTile;
      const int seg_end = u.start + u.len, kv_end = u.kvs + u.kvl;
      if (li == 0) {
        int ra[4], rb[4];
        fetch_rows(a.perm, u.start + u.q0, seg_end, u.h, ra);
        if (hb) fetch_rows(a.perm, u.start + u.q0 + kTile, seg_end, u.h, rb);
        if (!warp_wait(q_empty, (ucnt & 1) ^ 1, 1, ucnt)) { ok = false; break; }
        copy_tile(a.q, smem + P::kQA, ra, toks, u.len - u.q0, P::kChunkFull);
        if (hb) copy_tile(a.q, smem + P::kQB, rb, toks + kTile, u.len - u.q0 - kTile, P::kChunkFull);
        finish();
        if (lane == 0) mbar_arrive(q_full);
        ++ucnt;
        continue;
      }
      const bool is_v = li == 2;
      for (int j = 0; j < nkv; ++j, ++t) {
        int tr[4];
        // slot and phase in the ring of kStages tiles
        const int s = (int)(t % kStages);
        const uint32_t ph = t / kStages;
        fetch_rows(kvperm, u.kvs + j * kTile, kv_end, u.h, tr);
        if (!warp_wait(is_v ? &v_empty[s] : &k_empty[s], (ph & 1) ^ 1, is_v ? 3 : 2, t)) {
          ok = false;
          break;
        }
        // Test hook: the first K tile never arrives, so the MMA warp's
        // bounded wait runs out and the kernel reports a timeout.
        if (!is_v && t == 0 && a.debug_withhold_first_k) { ok = false; break; }
        uint8_t* dst = smem + (is_v ? P::kV0 : P::kK0) + s * P::kTileBytes;
        copy_tile(is_v ? a.v : a.k, dst, tr, toks, u.kvl - j * kTile, P::kChunkFull);
        finish();
        if (lane == 0) mbar_arrive(is_v ? &v_full[s] : &k_full[s]);
      }
    }
    // Row copies were waited for before their arrive, so nothing is in flight here.
  }
  if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, 128, false, false);
      constexpr uint32_t idO = idesc_bf16(128, DH, false, true);
      uint32_t ucnt = 0, kc = 0, vc = 0, pc0 = 0, pc1 = 0;
      bool ok = true;
      // S_x = Q_x K^T (both K-major in smem, 128B swizzle); qc / kch: byte
      // stride between the 64-column chunks of the query / key tile.
      auto issue_s = [&](int x, uint32_t qa, int qc, uint32_t ka, int kch) {
        const uint64_t qd = sdesc_sw128(qa, 16, 1024), kd = sdesc_sw128(ka, 16, 1024);
        const uint32_t ts = tS(x);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t qo = (kk >> 2) * qc + (kk & 3) * 32, ko = (kk >> 2) * kch + (kk & 3) * 32;
          umma_bf16(ts, sdesc_add(qd, qo), sdesc_add(kd, ko), idS, kk > 0 ? 1u : 0u);
        }
      };
      // O_x += P_x V (P in TMEM over S_x, V MN-major in smem, its 64-column
      // chunks kChunkFull bytes apart).
      auto issue_pv = [&](int x, uint32_t va, bool acc) {
        const uint64_t vd = sdesc_sw128(va, P::kChunkFull, 1024);
        const uint32_t to = tO(x), ts = tS(x);
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          umma_bf16_ts(to, ts + kk * 8, sdesc_add(vd, kk * 2048), idO, (acc || kk > 0) ? 1u : 0u);
      };
      // K/V tiles sit in a ring of kStages slots.
      auto kaddr = [&](int sl) { return smem_u32(smem + P::kK0 + sl * P::kTileBytes); };
      auto vaddr = [&](int sl) { return smem_u32(smem + P::kV0 + sl * P::kTileBytes); };
      const uint32_t qa_addr = smem_u32(smem + P::kQA), qb_addr = smem_u32(smem + P::kQB);
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        const Unit u = dec(idx);
        if (u.q0 >= u.len) continue;
        const bool hb = u.q0 + kTile < u.len;
        const int nkv = (u.kvl + kTile - 1) / kTile;
        if (!mbar_wait(q_full, ucnt & 1, wc, 4, ucnt)) break;
        ++ucnt;
        int ks = (int)(kc % kStages);
        if (!mbar_wait(&k_full[ks], (kc / kStages) & 1, wc, 5, kc)) break;
        tc_fence_after();
        issue_s(0, qa_addr, P::kChunkFull, kaddr(ks), P::kChunkFull);
        umma_commit(&s_full[0]);
        if (hb) {
          issue_s(1, qb_addr, P::kChunkFull, kaddr(ks), P::kChunkFull);
          umma_commit(&s_full[1]);
        }
        umma_commit(&k_empty[ks]);
        ++kc;
        if (nkv == 1) umma_commit(q_empty);
        for (int j = 0; j < nkv; ++j) {
          const int vs = (int)(vc % kStages);
          const bool more = j + 1 < nkv;
          ks = (int)(kc % kStages);
          // The next K tile is waited for before tile A's P, so that no wait
          // sits between tile A's P V and its next S (the loads do not depend
          // on P).
          if (!mbar_wait(&v_full[vs], (vc / kStages) & 1, wc, 7, vc)) { ok = false; break; }
          if (more && !mbar_wait(&k_full[ks], (kc / kStages) & 1, wc, 8, kc)) { ok = false; break; }
          if (!mbar_wait(&p_full[0], pc0 & 1, wc, 13, pc0)) { ok = false; break; }
          ++pc0;
          tc_fence_after();
          issue_pv(0, vaddr(vs), j > 0);
          if (more) {
            issue_s(0, qa_addr, P::kChunkFull, kaddr(ks), P::kChunkFull);
            umma_commit(&s_full[0]);
          } else {
            umma_commit(&o_full[0]);
          }
          if (hb) {
            if (!mbar_wait(&p_full[1], pc1 & 1, wc, 29, pc1)) { ok = false; break; }
            ++pc1;
            tc_fence_after();
            issue_pv(1, vaddr(vs), j > 0);
            if (more) {
              issue_s(1, qb_addr, P::kChunkFull, kaddr(ks), P::kChunkFull);
              umma_commit(&s_full[1]);
            } else {
              umma_commit(&o_full[1]);
            }
          }
          umma_commit(&v_empty[vs]);
          ++vc;
          if (more) {
            umma_commit(&k_empty[ks]);
            ++kc;
            if (j + 2 == nkv) umma_commit(q_empty);  // the unit's last S products are issued
          }
        }
      }
      umma_commit(done_bar);
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      mbar_wait(done_bar, 0, dc);
    }
  }
  } else {
    regs_inc<kRegsSoftmax>();
    // ---------------------------------------------------------------- softmax + epilogue
    const int x = (warp - 4) >> 2;  // warps 4-7: tile A, warps 8-11: tile B
    const int sub = warp & 3;       // TMEM sub-partition this warp may access
    const int row = sub * 32 + lane;
    const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
    const uint32_t tSx = tS(x) + lane_base, tOx = tO(x) + lane_base;
    const float scale_log2 = 1.4426950408889634f * rsqrtf((float)DH);
    uint32_t sc = 0, oc = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
      const Unit u = dec(idx);
      if (u.q0 >= u.len) continue;
      const bool hb = u.q0 + kTile < u.len;
      if (x == 1 && !hb) continue;
      const int nkv = (u.kvl + kTile - 1) / kTile;
      // The output row of this thread's query is fetched now, so its latency
      // hides behind the key loop.
      const int r = u.q0 + x * kTile + row;
      bool live = r < u.len;
      if (live && (u.h < 0 || u.h >= a.H || u.start < 0 || (int64_t)u.start + r >= N)) {  // outside the tensors
        live = false;
        if (status) atomicOr(status, DEV_RANGE);
      }
      const int src = live ? (a.perm ? a.perm[u.start + r] : u.start + r) : 0;
      float m_run = -INFINITY;
      uint64_t la = f2_pack(0.f, 0.f), lb = la, lc = la, ld = la;  // row sum of P, 8 partial sums
      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait(&s_full[x], sc & 1, wc, 6 + 16 * x, sc)) { ok = false; break; }
        ++sc;
        tc_fence_after();
        // The whole S row (128 fp32) is read from TMEM once.
        const int valid = u.kvl - j * kTile;  // keys of this tile inside the key/value segment
        float sr[kTile];
#pragma unroll
        for (int c = 0; c < kTile / 32; ++c) tmem_ld32(tSx + c * 32, sr + c * 32);
        tmem_ld_wait();
        if (valid < kTile) {  // only the segment's last KV tile has keys to mask
#pragma unroll
          for (int c = 0; c < kTile; ++c)
            if (c >= valid) sr[c] = -INFINITY;
        }
        // row max as a tree: 8 independent chains of 3-input maxima
        float m8[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          float m = fmax3(sr[16 * i], sr[16 * i + 1], sr[16 * i + 2]);
#pragma unroll
          for (int k = 3; k + 1 < 16; k += 2) m = fmax3(m, sr[16 * i + k], sr[16 * i + k + 1]);
          m8[i] = fmaxf(m, sr[16 * i + 15]);
        }
        const float mx = fmaxf(fmax3(m8[0], m8[1], m8[2]), fmax3(fmax3(m8[3], m8[4], m8[5]), m8[6], m8[7]));
        const float m_new = fmaxf(m_run, mx * scale_log2);
        // O_x was last written by the previous P V product, which completed
        // before this S (the MMA thread issued it first).  The running max is
        // moved (and O rescaled) only when it grows by more than 2^8; P and l
        // use the same stale max otherwise, so the result is unchanged.
        float alpha = 1.0f;
        bool rescale = false;
        if (j == 0) {
          m_run = m_new;
        } else {
          const bool need = m_new > m_run + 8.0f;
          rescale = __any_sync(0xffffffffu, need);
          if (need) {
            alpha = fast_exp2(m_run - m_new);
            const uint64_t a2 = f2_pack(alpha, alpha);
            la = f2_mul(la, a2);
            lb = f2_mul(lb, a2);
            lc = f2_mul(lc, a2);
            ld = f2_mul(ld, a2);
            m_run = m_new;
          }
        }
        // P = 2^(S*scale - m), summed into l and written back over S as packed
        // bf16 (two keys per TMEM column); pairs of keys go through the packed
        // fp32x2 FMA/ADD units.  Masked keys are -inf, so their P is 0.
        const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
        const uint64_t nm2 = f2_pack(-m_run, -m_run);
#pragma unroll
        for (int c = 0; c < kTile / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t t2 = f2_fma(f2_pack(sr[c * 32 + 2 * e], sr[c * 32 + 2 * e + 1]), sc2, nm2);
            float p0, p1;
            if (kExp2PolyEvery > 0 && e % (kExp2PolyEvery > 0 ? kExp2PolyEvery : 1) == kExp2PolyEvery - 1) {
              f2_unpack(exp2_poly_x2(t2), p0, p1);
            } else {
              float t0, t1;
              f2_unpack(t2, t0, t1);
              p0 = fast_exp2(t0);
              p1 = fast_exp2(t1);
            }
            const uint64_t pp = f2_pack(p0, p1);
            switch (e & 3) {
              case 0: la = f2_add(la, pp); break;
              case 1: lb = f2_add(lb, pp); break;
              case 2: lc = f2_add(lc, pp); break;
              default: ld = f2_add(ld, pp); break;
            }
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16u(tSx + c * 16, pk);
        }
        if (rescale) {
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            float o[32];
            tmem_ld32(tOx + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] *= alpha;
            tmem_st32(tOx + c * 32, o);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[x]);
      }
      if (!ok) break;
      // epilogue: wait for the last P V product, normalise, gate, scatter
      if (!mbar_wait(&o_full[x], oc & 1, wc, 9 + 16 * x, oc)) break;
      ++oc;
      tc_fence_after();
      if (live && (src < 0 || src >= N)) {
        live = false;
        if (status) atomicOr(status, DEV_RANGE);
      }
      float l_lo, l_hi;
      f2_unpack(f2_add(f2_add(la, lb), f2_add(lc, ld)), l_lo, l_hi);
      // log-sum-exp of the scaled scores: S*scale = log2(e)^-1 (m + log2 l)
      if (a.lse && live) a.lse[(int64_t)u.h * N + u.start + r] = (m_run + log2f(l_lo + l_hi)) * 0.6931471805599453f;
      const float gt = (live && a.gate) ? a.gate[src] : 1.0f;
      // output rows are written once: mark them first out of L2, so the K/V
      // tiles that other CTAs still read stay
      const uint64_t pol_out = l2_policy_evict_first();
      const float inv = a.out_scale * gt / (l_lo + l_hi);
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)src * a.H + u.h) * (int64_t)DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        float o[32];
        tmem_ld32(tOx + c * 32, o);
        tmem_ld_wait();
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            float w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = o[q4 * 8 + e] * inv;
            uint4 pk;
            pk.x = pack_bf16x2(w[0], w[1]);
            pk.y = pack_bf16x2(w[2], w[3]);
            pk.z = pack_bf16x2(w[4], w[5]);
            pk.w = pack_bf16x2(w[6], w[7]);
            // accumulate (a later branch of the block): out += this branch,
            // added by the memory system; otherwise a plain store.
            if (a.accumulate)
              red_add_bf16x8(dst + q4, pk);
            else
              st_global_hint(dst + q4, pk, pol_out);
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
  const uint64_t kv_rows = (uint64_t)(a.kv_rows > 0 ? a.kv_rows : a.N) * (uint64_t)a.H;
  // tiled: the gathered copies, Q [H*N rows, d_h] and K/V [H*kv_rows, d_h],
  // with 128-row boxes.  The in-place kernel copies rows itself and does not
  // read the maps.
  const uint32_t box_rows = (uint32_t)kTile;
  if (a.contiguous) {  // the caller's [N, H, d_h] tensors, read in place
    if (!make_tmap_tokens(&mq, a.q, DH, a.H, a.N) || !make_tmap_tokens(&mk, a.k, DH, a.H, a.N) ||
        !make_tmap_tokens(&mv, a.v, DH, a.H, a.N))
      return cudaErrorInvalidValue;
  } else {
    if (!make_tmap_2d(&mq, a.q, DH, rows, DH * 2, box_rows)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&mk, a.k, DH, kv_rows, DH * 2, box_rows)) return cudaErrorInvalidValue;
    if (!make_tmap_2d(&mv, a.v, DH, kv_rows, DH * 2, box_rows)) return cudaErrorInvalidValue;
  }
  // groups: the segment table; in place: the loaders' token rows (2 tiles each)
  const int table_ints = a.mode == 0 ? 3 * a.nseg + 1 : (a.direct ? 6 * kTile : 0);
  const size_t smem = P::bytes(table_ints);
  auto kern = a.direct ? attn_kernel<DH, true, true>
                       : (a.mode == 2 ? attn_kernel<DH, false, true> : attn_kernel<DH, false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = c.num_sms;
  if (a.mode == 1) {
    const int64_t tpw = ceil_div((int64_t)a.wt * a.wh * a.ww, kTile);
    const int64_t total = (int64_t)a.nseg * ((tpw + 1) / 2) * a.H;
    if (total < grid) grid = (int)total;
  }
  if (grid < 1) return cudaSuccess;
  kern<<<grid, kAttnThreads, smem, c.stream>>>(mq, mk, mv, a, c.status, (unsigned long long)c.wait_ns);
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

cudaError_t launch_gather_rows(const DevCtx& c, const void* a, const void* b, const int32_t* idx,
                               const int32_t* rows_dev, int64_t rows_max, int64_t N, int H, int d_h, int64_t stride,
                               void* da, void* db) {
  if (rows_max == 0) return cudaSuccess;
  int64_t blocks = ceil_div(rows_max, 8);
  const int64_t cap = (int64_t)c.num_sms * 8;
  if (blocks > cap) blocks = cap;
  gather_rows_kernel<<<(unsigned)blocks, 256, 0, c.stream>>>((const uint4*)a, (const uint4*)b, idx, rows_dev,
                                                             rows_max, N, H, d_h / 8, stride, (uint4*)da,
                                                             (uint4*)db, c.status);
  return cudaGetLastError();
}

cudaError_t launch_window_perm(const DevCtx& c, int T, int Hg, int Wg, const int* w, int32_t* perm_w) {
  const int N = T * Hg * Wg;
  if (N == 0) return cudaSuccess;
  WinGeom g{T, Hg, Wg, w[0], w[1], w[2], (int)ceil_div(Hg, w[1]), (int)ceil_div(Wg, w[2])};
  window_perm_kernel<<<(unsigned)ceil_div(N, 256), 256, 0, c.stream>>>(g, N, perm_w);
  return cudaGetLastError();
}

cudaError_t launch_seg_table(const DevCtx& c, const int32_t* offsets, int M, int H, int64_t N, int32_t* table,
                             int tiles_per_unit) {
  seg_table_kernel<<<1, 1024, 0, c.stream>>>(offsets, M, H, N, tiles_per_unit, table, c.status);
  return cudaGetLastError();
}

cudaError_t launch_attention(const DevCtx& c, const AttnArgs& a) {
  if (a.d_h == 128) return launch_attention_dh<128>(c, a);
  if (a.d_h == 64) return launch_attention_dh<64>(c, a);
  return cudaErrorInvalidValue;
}

}  // namespace moga
