// Gradients of the MoGA block (training): attention backward on tcgen05,
// the per-token preparation of dO and D, and the router backward.
//
// "MoGA: Mixture-of-Groups Attention for End-to-End Long Video Generation"
// (paper-graph-ui summary, section 3.4): the argmax assignment is not
// differentiable, so the router learns through the gate p(g(x)|x) that scales
// each token's group-attention output (Eq. 5, "Grouped Attention", "Gradient
// flow"); q, k, v receive the gradient of each branch's attention with the
// assignment held fixed.
//
// For one token set (a group or an STGA window) and one head, with
// S = Q K^T / sqrt(d_h), P = softmax(S), O = P V and dO the branch's share of
// the output gradient:
//   D_i = sum_c dO_ic O_ic,   dP = dO V^T,   dS = P * (dP - D),
//   dV = P^T dO,   dK = dS^T Q / sqrt(d_h),   dQ = dS K / sqrt(d_h).
// P is rebuilt from the forward's log-sum-exp: P_ij = exp(S_ij - lse_i).
//
// attn_bwd_kernel<DH, kDQ> is one persistent kernel shape for both halves:
// a CTA holds a 128-row "X" tile of one (segment, head) and streams the
// segment's 128-row "Y" tiles past it.
//   kDQ = false: X = (K, V) rows, Y = (Q, dO) rows:  S^T = K Q^T,
//                dP^T = V dO^T, then dV += P^T dO and dK += dS^T Q;
//   kDQ = true:  X = (Q, dO) rows, Y = (K, V) rows:  S = Q K^T, dP = dO V^T,
//                then dQ += dS K.
// Warp 0 loads tiles with TMA (and, for dK/dV, the per-column lse and D),
// warp 1 issues tcgen05.mma, warps 4-11 (two warpgroups, each owning 64 of
// the 128 Y columns of every TMEM lane) turn S and dP into bf16 P and dS in
// TMEM, which the accumulating products read as their A operand.
// S and dP each take a 128-column TMEM buffer.  The warpgroups read both
// into registers and write the packed bf16 operands (P and dS, or dS alone)
// into the S buffer, 64 columns at most, so the dP buffer is free as soon as
// dP is read.  dK/dV alternate two buffers (dV and dK fill the other 256
// columns): the next tile's S goes where dP was and is computed while the
// warpgroups finish this tile.  dQ keeps dP in one buffer and alternates S
// between two, issuing S a whole tile ahead (dQ takes the last 128).  Y1 (Q or K) sits in a three-slot ring, since the
// closing product reads it a tile after S did; Y2 (dO or V) in two slots.
// 128-row Y tiles are the faster choice, because an M=128 MMA reads its
// whole A slice from shared memory for every instruction, and N = 128
// halves those bytes per multiply-add against N = 64 (shared-memory
// bandwidth bounds those products).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>

#include "internal.h"
#include "ptx.cuh"
#include "windows.cuh"

namespace moga {
namespace {

constexpr int kBwdThreads = 384;
constexpr int kYRows = 128;
constexpr float kLog2e = 1.4426950408889634f;

template <int DH, bool kDQ>
struct BPlan {
  static constexpr int kChunks = DH / 64;
  static constexpr int kXBytes = kTile * DH * 2;    // 128-row bf16 tile
  static constexpr int kYBytes = kYRows * DH * 2;   // 128-row bf16 tile
  static constexpr int kXChunk = kTile * 128;       // bytes of one 64-column chunk of an X tile
  static constexpr int kYChunk = kYRows * 128;      // the same for a Y tile
  // Y1 and Y2 tiles sit in rings of their own.  Y1 (Q, or K for dQ) is
  // read by S in its tile's turn and by the product that closes the tile
  // (dK += dS^T Q, or dQ += dS K) during the next tile's, so its ring has
  // three slots; Y2 (dO, or V) is first read by dP, later in its tile's
  // turn, and two slots keep it ahead.
  static constexpr int kS1 = 3;
  static constexpr int kS2 = 2;
  static constexpr int kX1 = 0;
  static constexpr int kX2 = kXBytes;
  static constexpr int kY1 = 2 * kXBytes;
  static constexpr int kY2 = kY1 + kS1 * kYBytes;
  // dK/dV: -lse*log2(e) of the Y rows per Y1 slot and D per Y2 slot (fp32)
  static constexpr int kVec1 = kY2 + kS2 * kYBytes;
  static constexpr int kVec2 = kVec1 + (kDQ ? 0 : kS1 * kYRows * 4);
  static constexpr int kBar = kVec2 + (kDQ ? 0 : kS2 * kYRows * 4);
  static constexpr int kTable = kBar + 256;
};

struct BUnit {
  int h, start, len, x0;  // segment [start, start + len) of head h; X tile rows [x0, x0 + 128)
};

struct BDecoder {
  int mode;        // 0 groups (table), 1 windows (geometry)
  int nseg;
  const int* tab;  // [unit_prefix (M+1) | seg_start (M) | seg_len (M)]: a shared copy, or global
  WinGeom g;
  int upw;         // windows: X tiles per window
  __device__ __forceinline__ BUnit operator()(int idx) const {
    BUnit u;
    if (mode == 0) {
      int lo = 0, hi = nseg - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tab[mid] <= idx) lo = mid; else hi = mid - 1;
      }
      const int local = idx - tab[lo];
      u.start = tab[nseg + 1 + lo];
      u.len = tab[2 * nseg + 1 + lo];
      const int nt = (u.len + kTile - 1) / kTile;
      u.h = local / nt;
      u.x0 = (local - u.h * nt) * kTile;
    } else {
      const int xt = idx % upw;
      const int rest = idx / upw;
      const int seg = rest % nseg;
      u.h = rest / nseg;
      window_of(g, seg, u.start, u.len);
      u.x0 = xt * kTile;
    }
    return u;
  }
};

// tab_smem: copy the segment table into shared memory (it fits); pad: bytes
// allocated beyond the plan, for aligning the tiles to 1024 B.
template <int DH, bool kDQ>
__global__ void __launch_bounds__(kBwdThreads, 1)
attn_bwd_kernel(const __grid_constant__ CUtensorMap tx1, const __grid_constant__ CUtensorMap tx2,
                const __grid_constant__ CUtensorMap ty1, const __grid_constant__ CUtensorMap ty2, const BwdArgs a,
                int tab_smem, int pad, int* status, unsigned long long wait_ns) {
  using P = BPlan<DH, kDQ>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t off = ((raw + 1023u) & ~1023u) - raw;
  if (off > (uint32_t)pad) {  // no room to align the swizzled tiles: the whole CTA returns at once
    if (threadIdx.x == 0 && status) atomicOr(status, DEV_RANGE);
    return;
  }
  uint8_t* smem = smem_raw + off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::kBar);
  uint64_t* x_full = bars + 0;
  uint64_t* x_empty = bars + 1;
  uint64_t* y1_full = bars + 2;                 // [kS1]
  uint64_t* y1_empty = y1_full + P::kS1;        // [kS1]
  uint64_t* y2_full = y1_empty + P::kS1;        // [kS2]
  uint64_t* y2_empty = y2_full + P::kS2;        // [kS2]
  uint64_t* s_full = y2_empty + P::kS2;         // [2]: S computed (dQ: S(t) on s_full[t % 2])
  uint64_t* d_full = s_full + 2;                // dP computed
  // [2]: P and dS of tile t written, on p_full[t % 2].  Two barriers,
  // because the dQ pass issues dP(t + 1) before it waits for tile t, so the
  // warpgroups may finish tile t + 1 before that wait begins; the next phase
  // of the same barrier needs dP(t + 2), which comes after it.
  uint64_t* p_full = d_full + 1;
  uint64_t* acc_full = p_full + 2;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* dp_free = acc_empty + 1;            // the warpgroups have read dP
  uint64_t* done_bar = dp_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(done_bar + 2);
  static_assert(2 + 2 * (P::kS1 + P::kS2) + 11 <= 32, "barrier area holds 32 words");
  int* tab = reinterpret_cast<int*>(smem + P::kTable);
  float* vec1 = reinterpret_cast<float*>(smem + P::kVec1);
  float* vec2 = reinterpret_cast<float*>(smem + P::kVec2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(x_full, 1);
    mbar_init(x_empty, 1);
    // dK/dV: the TMA bytes and the lse (Y1) or D (Y2) vector
    for (int s = 0; s < P::kS1; ++s) {
      mbar_init(&y1_full[s], kDQ ? 1 : 2);
      mbar_init(&y1_empty[s], 1);
    }
    for (int s = 0; s < P::kS2; ++s) {
      mbar_init(&y2_full[s], kDQ ? 1 : 2);
      mbar_init(&y2_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(d_full, 1);
    mbar_init(&p_full[0], 256);
    mbar_init(&p_full[1], 256);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 256);
    mbar_init(dp_free, 256);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  BDecoder dec;
  dec.mode = a.mode;
  dec.nseg = a.nseg;
  dec.tab = a.table;
  dec.upw = 1;
  if (a.mode == 0) {
    if (tab_smem) {
      const int n = 3 * a.nseg + 1;
      for (int i = threadIdx.x; i < n; i += blockDim.x) tab[i] = a.table[i];
      dec.tab = tab;
    }
  } else {
    dec.g = WinGeom{a.T, a.Hg, a.Wg, a.wt, a.wh, a.ww, (a.Hg + a.wh - 1) / a.wh, (a.Wg + a.ww - 1) / a.ww};
    dec.upw = (a.wt * a.wh * a.ww + kTile - 1) / kTile;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int total = a.mode == 0 ? dec.tab[a.nseg] : a.nseg * dec.upw * a.H;
  const uint32_t tmem = *tmem_slot;
  const uint32_t tAccA = tmem + 256u;                // dV, or dQ
  const uint32_t tAccB = tmem + 256u + (uint32_t)DH; // dK
  // TMEM buffers of Y tile yc (a CTA-wide tile counter).  S goes to one
  // 128-column buffer and dP to another; the warpgroups read both into
  // registers and write the packed bf16 operands of the closing products
  // (dK/dV: P, then dS 32 columns further; dQ: dS) into the S buffer.  So
  // the dP buffer is free once dP is read.
  //   dK/dV: two buffers (0, 128; dV and dK fill the rest) swap roles:
  //          S(yc) in buffer yc % 2, dP(yc) in the other, which held the
  //          previous tile's S (its P and dS are read before dP(yc) is
  //          issued); S(yc + 1) is computed while the warpgroups finish yc.
  //   dQ:    S alternates between 0 and 384, dP stays at 128 (dQ at 256).
  //          S(yc + 1) is issued right after dQ(yc - 1) has read dS from
  //          its buffer, a whole tile ahead, and dP(yc + 1) once dP(yc) is
  //          read.
  auto tSb = [&](uint32_t yc_) { return kDQ ? tmem + ((yc_ & 1u) ? 384u : 0u) : tmem + 128u * (yc_ & 1u); };
  auto tDb = [&](uint32_t yc_) { return kDQ ? tmem + 128u : tmem + 128u * ((yc_ & 1u) ^ 1u); };
  WaitCtx wc{abort_flag, status, wait_ns};
  const int64_t N = a.N;

  if (warp == 0) {
    // ---------------------------------------------------------------- loads
    uint32_t uc = 0, n1 = 0, n2 = 0;  // X tiles, Y1 and Y2 tiles issued
    bool ok = true;
    auto wwait = [&](uint64_t* bar, uint32_t parity, int site, uint32_t count) {
      int w = 1;
      if (lane == 0) w = mbar_wait(bar, parity, wc, site, count);
      return __shfl_sync(0xffffffffu, w, 0) != 0;
    };
    if (lane == 0) {
      tma_prefetch_desc(&tx1);
      tma_prefetch_desc(&tx2);
      tma_prefetch_desc(&ty1);
      tma_prefetch_desc(&ty2);
    }
    // dK/dV: this lane's share of a Y tile's -lse*log2(e) and D, read one
    // tile ahead so that their latency hides behind the rings' waits.  Rows
    // past the segment get -inf and 0, so their P and dS are exactly 0.
    float lv[kYRows / 32], dv[kYRows / 32];
    auto fetch = [&](const BUnit& u, int i) {
#pragma unroll
      for (int q = 0; q < kYRows / 32; ++q) {
        const int pos = i * kYRows + lane + 32 * q;
        const bool valid = pos < u.len;
        const int64_t gi = (int64_t)u.h * N + u.start + pos;
        lv[q] = valid ? -a.lse[gi] * kLog2e : -INFINITY;
        dv[q] = valid ? a.dsum[gi] : 0.0f;
      }
    };
    // plain shared-memory stores of a vector, then the slot's second arrival
    auto put = [&](float* v, const float* r, uint64_t* bar) {
#pragma unroll
      for (int q = 0; q < kYRows / 32; ++q) v[lane + 32 * q] = r[q];
      __threadfence_block();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar);
    };
    for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
      const BUnit u = dec(idx);
      if (u.x0 >= u.len) continue;
      const int ny = (u.len + kYRows - 1) / kYRows;
      if (!wwait(x_empty, (uc & 1) ^ 1, 1, uc)) break;
      if (lane == 0) {
        const int row = (int)((int64_t)u.h * N + u.start + u.x0);
        mbar_expect_tx(x_full, 2 * P::kXBytes);
#pragma unroll
        for (int c = 0; c < P::kChunks; ++c) {
          tma_load_2d(&tx1, x_full, smem + P::kX1 + c * P::kXChunk, c * 64, row);
          tma_load_2d(&tx2, x_full, smem + P::kX2 + c * P::kXChunk, c * 64, row);
        }
      }
      ++uc;
      if (!kDQ) fetch(u, 0);
      for (int i = 0; i < ny; ++i) {
        const int row = (int)((int64_t)u.h * N + u.start + i * kYRows);
        const int s1 = (int)(n1 % P::kS1);
        if (!wwait(&y1_empty[s1], ((n1 / P::kS1) & 1) ^ 1, 2, n1)) { ok = false; break; }
        if (lane == 0) {
          uint8_t* y = smem + P::kY1 + s1 * P::kYBytes;
          mbar_expect_tx(&y1_full[s1], P::kYBytes);
#pragma unroll
          for (int c = 0; c < P::kChunks; ++c) tma_load_2d(&ty1, &y1_full[s1], y + c * P::kYChunk, c * 64, row);
        }
        if (!kDQ) put(vec1 + s1 * kYRows, lv, &y1_full[s1]);
        ++n1;
        const int s2 = (int)(n2 % P::kS2);
        if (!wwait(&y2_empty[s2], ((n2 / P::kS2) & 1) ^ 1, 16, n2)) { ok = false; break; }
        if (lane == 0) {
          uint8_t* y = smem + P::kY2 + s2 * P::kYBytes;
          mbar_expect_tx(&y2_full[s2], P::kYBytes);
#pragma unroll
          for (int c = 0; c < P::kChunks; ++c) tma_load_2d(&ty2, &y2_full[s2], y + c * P::kYChunk, c * 64, row);
        }
        if (!kDQ) {
          put(vec2 + s2 * kYRows, dv, &y2_full[s2]);
          if (i + 1 < ny) fetch(u, i + 1);
        }
        ++n2;
      }
    }
    // Drain every load this warp issued before the CTA exits.
    if (lane == 0) {
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      if (uc > 0) mbar_wait(x_full, (uc - 1) & 1, dc);
      for (int s = 0; s < P::kS1; ++s)
        if ((uint32_t)s < n1) mbar_wait(&y1_full[s], ((n1 - 1 - ((n1 - 1 - s) % P::kS1)) / P::kS1) & 1, dc);
      for (int s = 0; s < P::kS2; ++s)
        if ((uint32_t)s < n2) mbar_wait(&y2_full[s], ((n2 - 1 - ((n2 - 1 - s) % P::kS2)) / P::kS2) & 1, dc);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, kYRows, false, false);
      constexpr uint32_t idA = idesc_bf16(128, DH, false, true);
      const uint32_t x1 = smem_u32(smem + P::kX1), x2 = smem_u32(smem + P::kX2);
      uint32_t uc = 0, yc = 0;
      bool ok = true;
      // S (or S^T) = X1 Y1^T and dP (or dP^T) = X2 Y2^T, both operands K-major.
      const uint64_t x1d = sdesc_sw128(x1, 16, 1024), x2d = sdesc_sw128(x2, 16, 1024);
      // S and dP with their own commits, so that the softmax warps compute
      // P while the tensor core computes dP.
      auto issue_sonly = [&](uint32_t ycs) {
        const uint64_t y1d = sdesc_sw128(smem_u32(smem + P::kY1 + (ycs % P::kS1) * P::kYBytes), 16, 1024);
        const uint32_t ts = tSb(ycs);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t xo = (kk >> 2) * P::kXChunk + (kk & 3) * 32, yo = (kk >> 2) * P::kYChunk + (kk & 3) * 32;
          umma_bf16(ts, sdesc_add(x1d, xo), sdesc_add(y1d, yo), idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[kDQ ? (ycs & 1u) : 0u]);
      };
      auto issue_dp = [&](uint32_t ycs) {
        const uint64_t y2d = sdesc_sw128(smem_u32(smem + P::kY2 + (ycs % P::kS2) * P::kYBytes), 16, 1024);
        const uint32_t td = tDb(ycs);
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t xo = (kk >> 2) * P::kXChunk + (kk & 3) * 32, yo = (kk >> 2) * P::kYChunk + (kk & 3) * 32;
          umma_bf16(td, sdesc_add(x2d, xo), sdesc_add(y2d, yo), idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(d_full);
      };
      // Accumulations over the 128 Y rows (eight 16-row steps).  Warpgroup w
      // wrote P / dS of Y rows [64w, 64w + 64) as packed bf16 into the S
      // buffer, 32 columns from 64w (dK/dV: P there, dS 32 columns further),
      // so step kk's 16 rows start at column 64 (kk / 4) + 8 (kk % 4).
      auto issue_acc = [&](uint32_t ycs, bool acc) {
        const uint64_t y1d = sdesc_sw128(smem_u32(smem + P::kY1 + (ycs % P::kS1) * P::kYBytes), P::kYChunk, 1024);
        const uint64_t y2d = sdesc_sw128(smem_u32(smem + P::kY2 + (ycs % P::kS2) * P::kYBytes), P::kYChunk, 1024);
        const uint32_t ts = tSb(ycs);
#pragma unroll
        for (int kk = 0; kk < kYRows / 16; ++kk) {
          const uint32_t pc = 64u * (kk >> 2) + 8u * (kk & 3);
          const uint32_t en = (acc || kk > 0) ? 1u : 0u;
          if (kDQ) {
            umma_bf16_ts(tAccA, ts + pc, sdesc_add(y1d, kk * 2048), idA, en);  // dQ += dS K
          } else {
            umma_bf16_ts(tAccA, ts + pc, sdesc_add(y2d, kk * 2048), idA, en);       // dV += P^T dO
            umma_bf16_ts(tAccB, ts + 32 + pc, sdesc_add(y1d, kk * 2048), idA, en);  // dK += dS^T Q
          }
        }
      };
      // Tile t's accumulations, once the warpgroups have written its P and
      // dS (and, for a unit's first tile, read out the previous unit's
      // accumulators); they are the last readers of its Y1 tile (and, for
      // dK/dV, of its Y2 tile).
      auto finish_tile = [&](uint32_t t, bool first, bool last_of_unit) {
        if (!mbar_wait(&p_full[t & 1], (t >> 1) & 1, wc, 5, t)) return false;
        if (first && uc > 0 && !mbar_wait(acc_empty, (uc - 1) & 1, wc, 6, uc)) return false;
        tc_fence_after();
        issue_acc(t, !first);
        umma_commit(&y1_empty[t % P::kS1]);
        if (!kDQ) umma_commit(&y2_empty[t % P::kS2]);
        if (last_of_unit) umma_commit(acc_full);
        return true;
      };
      auto wait_y1 = [&](uint32_t t) { return mbar_wait(&y1_full[t % P::kS1], (t / P::kS1) & 1, wc, 4, t); };
      auto wait_y2 = [&](uint32_t t) { return mbar_wait(&y2_full[t % P::kS2], (t / P::kS2) & 1, wc, 17, t); };
      for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
        const BUnit u = dec(idx);
        if (u.x0 >= u.len) continue;
        const int ny = (u.len + kYRows - 1) / kYRows;
        if (!mbar_wait(x_full, uc & 1, wc, 3, uc)) break;
        if (kDQ) {
          // Order per tile: dP(i), dQ(i-1), S(i+1).  dP(i) goes where dP(i-1)
          // was, once the warpgroups have read it; S(i+1) where S(i-1) was,
          // after dQ(i-1) read its dS (the tensor pipe runs in issue order).
          // V is read by dP alone and released right after it.
          if (!wait_y1(yc)) break;
          tc_fence_after();
          issue_sonly(yc);
          for (int i = 0; i < ny; ++i) {
            if (!wait_y2(yc)) { ok = false; break; }
            if (yc > 0 && !mbar_wait(dp_free, (yc - 1) & 1, wc, 15, yc)) { ok = false; break; }
            tc_fence_after();
            issue_dp(yc);
            umma_commit(&y2_empty[yc % P::kS2]);
            if (i + 1 == ny) umma_commit(x_empty);
            if (i > 0 && !finish_tile(yc - 1, i == 1, false)) { ok = false; break; }
            if (i + 1 < ny) {
              if (!wait_y1(yc + 1)) { ok = false; break; }
              tc_fence_after();
              issue_sonly(yc + 1);
            }
            ++yc;
          }
        } else {
          // Order per tile: S(i), dV/dK(i-1), dP(i).  S(i) goes where dP(i-1)
          // was, once the warpgroups have read it; dP(i) where dV/dK(i-1)
          // read P and dS of tile i-1 just before (the tensor pipe runs in
          // issue order).
          for (int i = 0; i < ny; ++i) {
            if (!wait_y1(yc)) { ok = false; break; }
            if (yc > 0 && !mbar_wait(dp_free, (yc - 1) & 1, wc, 15, yc)) { ok = false; break; }
            tc_fence_after();
            issue_sonly(yc);
            if (i > 0 && !finish_tile(yc - 1, i == 1, false)) { ok = false; break; }
            if (!wait_y2(yc)) { ok = false; break; }
            tc_fence_after();
            issue_dp(yc);
            if (i + 1 == ny) umma_commit(x_empty);
            ++yc;
          }
        }
        if (!ok || !finish_tile(yc - 1, ny == 1, true)) break;
        ++uc;
      }
      umma_commit(done_bar);
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      mbar_wait(done_bar, 0, dc);
    }
  } else if (warp >= 4) {
    // ---------------------------------------------------------------- P, dS and the epilogue
    const int wg = (warp - 4) >> 2;   // Y columns [64 wg, 64 wg + 64) of every tile
    const int sub = warp & 3;         // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;  // X row = TMEM lane
    const uint32_t lb = (uint32_t)(sub * 32) << 16;
    const float scale_log2 = kLog2e * rsqrtf((float)DH);
    const float scale = rsqrtf((float)DH);
    uint32_t uc = 0, yc = 0;
    bool ok = true;
    for (int idx = blockIdx.x; idx < total && ok; idx += gridDim.x) {
      const BUnit u = dec(idx);
      if (u.x0 >= u.len) continue;
      const int ny = (u.len + kYRows - 1) / kYRows;
      const int r = u.x0 + row;
      bool live = r < u.len;
      if (live && (u.h < 0 || u.h >= a.H || u.start < 0 || (int64_t)u.start + r >= N)) {
        live = false;
        if (status) atomicOr(status, DEV_RANGE);
      }
      float nl_row = -INFINITY, d_row = 0.0f;  // dQ: this query row's -lse*log2(e) and D
      if (kDQ && live) {
        const int64_t gi = (int64_t)u.h * N + u.start + r;
        nl_row = -a.lse[gi] * kLog2e;
        d_row = a.dsum[gi];
      }
      const int src = live ? (a.perm ? a.perm[u.start + r] : u.start + r) : 0;
      for (int i = 0; i < ny; ++i, ++yc) {
        const int s1 = (int)(yc % P::kS1), s2 = (int)(yc % P::kS2);
        // dQ: S(t) on s_full[t % 2], whose phase advances every other tile
        // (S runs a tile ahead); dK/dV: s_full[0]
        const bool ok_s = kDQ ? mbar_wait(&s_full[yc & 1], (yc >> 1) & 1, wc, 7 + wg, yc)
                              : mbar_wait(&s_full[0], yc & 1, wc, 7 + wg, yc);
        if (!ok_s) { ok = false; break; }
        tc_fence_after();
        // the vectors are plain shared-memory stores of the load warp: wait
        // on the slot's own barrier too (its phase is still this tile's,
        // since the slot is refilled only after this tile's P and dS)
        if (!kDQ && !mbar_wait(&y1_full[s1], (yc / P::kS1) & 1, wc, 11 + wg, yc)) { ok = false; break; }
        // Y columns [64 wg, 64 wg + 64): P from S as soon as S is in (the
        // tensor core is still computing dP), then dS once dP is in.  The
        // packed P (dK/dV) and dS of half hf go to S-buffer columns
        // 64 wg + 16 hf and, for dK/dV's dS, 32 further: columns this
        // warpgroup has already read.
        const uint32_t ts = tSb(yc), td = tDb(yc);
        float pv[64];
        {
          float sv[64];
          tmem_ld32(ts + lb + 64 * wg, sv);
          tmem_ld32(ts + lb + 64 * wg + 32, sv + 32);
          tmem_ld_wait();
          if (kDQ) {
            const int valid = u.len - i * kYRows - 64 * wg;  // keys of these columns inside the segment
#pragma unroll
            for (int e = 0; e < 64; ++e) {
              const float pe = fast_exp2(fmaf(sv[e], scale_log2, nl_row));
              pv[e] = e < valid ? pe : 0.0f;
            }
          } else {
            // the slot's -lse*log2(e), read as 16-byte vectors (one broadcast
            // wavefront per four keys)
            const float4* nl = reinterpret_cast<const float4*>(vec1 + s1 * kYRows + 64 * wg);
#pragma unroll
            for (int e4 = 0; e4 < 16; ++e4) {
              const float4 n = nl[e4];
              pv[4 * e4 + 0] = fast_exp2(fmaf(sv[4 * e4 + 0], scale_log2, n.x));
              pv[4 * e4 + 1] = fast_exp2(fmaf(sv[4 * e4 + 1], scale_log2, n.y));
              pv[4 * e4 + 2] = fast_exp2(fmaf(sv[4 * e4 + 2], scale_log2, n.z));
              pv[4 * e4 + 3] = fast_exp2(fmaf(sv[4 * e4 + 3], scale_log2, n.w));
            }
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              uint32_t pk[16];
#pragma unroll
              for (int e = 0; e < 16; ++e) pk[e] = pack_bf16x2(pv[32 * hf + 2 * e], pv[32 * hf + 2 * e + 1]);
              tmem_st16u(ts + lb + 64 * wg + 16 * hf, pk);
            }
          }
        }
        if (!mbar_wait(d_full, yc & 1, wc, 13 + wg, yc)) { ok = false; break; }
        tc_fence_after();
        {
          // all of dP is read first, so its buffer is released for the next
          // tile's S before dS is computed
          float dv[64];
          tmem_ld32(td + lb + 64 * wg, dv);
          tmem_ld32(td + lb + 64 * wg + 32, dv + 32);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(dp_free);
          // D per Y row (dK/dV: from the Y2 slot's vector), or of this X row (dQ)
          const float4* dd = reinterpret_cast<const float4*>(vec2 + s2 * kYRows + 64 * wg);
          if (!kDQ && !mbar_wait(&y2_full[s2], (yc / P::kS2) & 1, wc, 18 + wg, yc)) { ok = false; break; }
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            uint32_t dk[16];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {
              const int c = 32 * hf + 2 * e;
              if (kDQ) {
                dk[e] = pack_bf16x2(pv[c] * (dv[c] - d_row), pv[c + 1] * (dv[c + 1] - d_row));
                dk[e + 1] = pack_bf16x2(pv[c + 2] * (dv[c + 2] - d_row), pv[c + 3] * (dv[c + 3] - d_row));
              } else {
                const float4 D = dd[c >> 2];
                dk[e] = pack_bf16x2(pv[c] * (dv[c] - D.x), pv[c + 1] * (dv[c + 1] - D.y));
                dk[e + 1] = pack_bf16x2(pv[c + 2] * (dv[c + 2] - D.z), pv[c + 3] * (dv[c + 3] - D.w));
              }
            }
            tmem_st16u(ts + lb + 64 * wg + (kDQ ? 0 : 32) + 16 * hf, dk);
          }
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[yc & 1]);
      }
      if (!ok) break;
      // ------------------------------------------------ epilogue
      if (!mbar_wait(acc_full, uc & 1, wc, 9 + wg, uc)) break;
      ++uc;
      tc_fence_after();
      if (live && (src < 0 || src >= N)) {
        live = false;
        if (status) atomicOr(status, DEV_RANGE);
      }
      // dK/dV: warpgroup 0 writes dV, warpgroup 1 dK (scaled); dQ: each
      // warpgroup writes half of the columns (scaled).
      uint32_t tacc;
      void* outp;
      int c0, nc;
      float f;
      if (kDQ) {
        tacc = tAccA + (uint32_t)(wg * DH / 2);
        outp = a.out1;
        c0 = wg * DH / 2;
        nc = DH / 2;
        f = scale;
      } else {
        tacc = wg ? tAccB : tAccA;
        outp = wg ? a.out2 : a.out1;
        c0 = 0;
        nc = DH;
        f = wg ? scale : 1.0f;
      }
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(outp) + ((int64_t)src * a.H + u.h) * (int64_t)DH + c0;
      for (int c = 0; c < nc / 32; ++c) {
        float o[32];
        tmem_ld32(tacc + lb + c * 32, o);
        tmem_ld_wait();
        if (live) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            uint4 pk;
            pk.x = pack_bf16x2(o[q4 * 8 + 0] * f, o[q4 * 8 + 1] * f);
            pk.y = pack_bf16x2(o[q4 * 8 + 2] * f, o[q4 * 8 + 3] * f);
            pk.z = pack_bf16x2(o[q4 * 8 + 4] * f, o[q4 * 8 + 5] * f);
            pk.w = pack_bf16x2(o[q4 * 8 + 6] * f, o[q4 * 8 + 7] * f);
            if (a.accumulate)
              red_add_bf16x8(dst + q4, pk);
            else
              dst[q4] = pk;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DH, bool kDQ>
cudaError_t launch_bwd_dh(const DevCtx& c, const BwdArgs& a) {
  using P = BPlan<DH, kDQ>;
  CUtensorMap m1, m2, m3, m4;
  const uint64_t rows = (uint64_t)a.N * (uint64_t)a.H;
  // X and Y: 128-row boxes (all [H][N][d_h] head-major copies)
  const void* xs1 = kDQ ? a.q : a.k;
  const void* xs2 = kDQ ? a.dout : a.v;
  const void* ys1 = kDQ ? a.k : a.q;
  const void* ys2 = kDQ ? a.v : a.dout;
  if (!make_tmap_2d(&m1, xs1, DH, rows, DH * 2, kTile) || !make_tmap_2d(&m2, xs2, DH, rows, DH * 2, kTile) ||
      !make_tmap_2d(&m3, ys1, DH, rows, DH * 2, kYRows) || !make_tmap_2d(&m4, ys2, DH, rows, DH * 2, kYRows))
    return cudaErrorInvalidValue;
  // the device's opt-in shared memory per block, queried once per device
  static std::atomic<int> cached[64];
  int max_smem = (c.device >= 0 && c.device < 64) ? cached[c.device].load(std::memory_order_relaxed) : 0;
  cudaError_t e = cudaSuccess;
  if (max_smem <= 0) {
    if ((e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, c.device)) != cudaSuccess)
      return e;
    if (c.device >= 0 && c.device < 64) cached[c.device].store(max_smem, std::memory_order_relaxed);
  }
  // The segment table goes to shared memory when it fits beside the tiles
  // (the kernel reads it from global memory otherwise); up to 1 KB more
  // aligns the tiles to 1024 B, and the kernel checks that it got enough.
  const size_t table_bytes = a.mode == 0 ? (size_t)(3 * a.nseg + 1) * 4 : 0;
  const bool tab_smem = P::kTable + table_bytes <= (size_t)max_smem;
  const size_t need = P::kTable + (tab_smem ? table_bytes : 0);
  if (need > (size_t)max_smem) return cudaErrorInvalidValue;
  const size_t smem = std::min(need + 1024, (size_t)max_smem);
  auto kern = attn_bwd_kernel<DH, kDQ>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int grid = c.num_sms;
  if (a.mode == 1) {
    const int64_t total = (int64_t)a.nseg * ceil_div((int64_t)a.wt * a.wh * a.ww, kTile) * a.H;
    if (total < grid) grid = (int)total;
  }
  if (grid < 1) return cudaSuccess;
  kern<<<grid, kBwdThreads, smem, c.stream>>>(m1, m2, m3, m4, a, tab_smem ? 1 : 0, (int)(smem - need), c.status,
                                              (unsigned long long)c.wait_ns);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ dO, D and the gate gradient
// One warp per segment position j (token src = perm[j]), all heads:
//   dO_hat[h][j] = w * gate[src] * dout[src, h]          (bf16, head-major)
//   D[h][j]      = w * sum_c dout[src, h, c] * o[src, h, c]
//   dgate[src]   = sum_h D[h][j] / gate[src]              (when dgate is given)
// where o is the branch's output as the forward stored it (for MoGA the
// gated output gate * SA, so D equals sum_c dO_hat * SA).
__global__ void __launch_bounds__(256)
bwd_prep_kernel(const uint4* __restrict__ dout, const uint4* __restrict__ o, const int32_t* __restrict__ perm,
                const float* __restrict__ gate, float w, int64_t N, int H, int vph, uint4* __restrict__ dO_hat,
                float* __restrict__ dsum, float* __restrict__ dgate, int* status) {
  const int lane = threadIdx.x & 31;
  const int64_t w0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int64_t nw = ((int64_t)gridDim.x * blockDim.x) >> 5;
  const int vpr = H * vph;
  const int iters = (vpr + 31) / 32;
  for (int64_t j = w0; j < N; j += nw) {
    const int64_t src = perm ? perm[j] : j;
    if (src < 0 || src >= N) {
      if (lane == 0 && status) atomicOr(status, DEV_RANGE);
      continue;
    }
    const float g = gate ? gate[src] : 1.0f;
    const float sc = w * g;
    float dg = 0.0f;
    for (int it = 0; it < iters; ++it) {
      const int u = it * 32 + lane;
      const bool act = u < vpr;
      const int h = u / vph, c = u - h * vph;
      float part = 0.0f;
      if (act) {
        const uint4 dv = dout[src * vpr + u];
        const uint4 ov = o[src * vpr + u];
        const __nv_bfloat162* d2 = reinterpret_cast<const __nv_bfloat162*>(&dv);
        const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 df = __bfloat1622float2(d2[e]);
          const float2 of = __bfloat1622float2(o2[e]);
          part = fmaf(df.x, of.x, part);
          part = fmaf(df.y, of.y, part);
          pk[e] = pack_bf16x2(df.x * sc, df.y * sc);
        }
        dO_hat[((int64_t)h * N + j) * vph + c] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
      for (int off = vph >> 1; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
      if (act && c == 0) {
        dsum[(int64_t)h * N + j] = w * part;
        dg += w * part;
      }
    }
    if (dgate) {
      for (int off = 16; off > 0; off >>= 1) dg += __shfl_xor_sync(0xffffffffu, dg, off);
      if (lane == 0) dgate[src] = dg / g;
    }
  }
}

// out = (x + y (+ z)) / (2 or 3), bf16, n8 groups of 8 values (z nullable)
__global__ void __launch_bounds__(256) mean_kernel(const uint4* __restrict__ x, const uint4* __restrict__ y,
                                                   const uint4* __restrict__ z, int64_t n8, uint4* __restrict__ out) {
  const float inv = z ? (1.0f / 3.0f) : 0.5f;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 a = x[i], b = y[i];
    const uint4 c = z ? z[i] : make_uint4(0, 0, 0, 0);
    const __nv_bfloat162* a2 = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* b2 = reinterpret_cast<const __nv_bfloat162*>(&b);
    const __nv_bfloat162* c2 = reinterpret_cast<const __nv_bfloat162*>(&c);
    uint32_t pk[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 fa = __bfloat1622float2(a2[e]), fb = __bfloat1622float2(b2[e]), fc = __bfloat1622float2(c2[e]);
      pk[e] = pack_bf16x2(inv * (fa.x + fb.x + fc.x), inv * (fa.y + fb.y + fc.y));
    }
    out[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
}

// ------------------------------------------------------------------ router backward
// Eqs. 2-3 ("MoGA Router") differentiated through the gate:
//   r = x W_r^T + b,  p = softmax(r),  gate = p_g (g = the forward's group id),
//   dr_j = dgate * p_g * ([j == g] - p_j)
//        + bcoef * p_j * (F_j - sum_k F_k p_k)   (the group balancing loss of
//          Eq. 6, alpha * M * sum_i F_i P_i with P_i the mean of p(i|x) over
//          the N tokens: bcoef = alpha * M / N; F_i, the share of tokens routed
//          to i, comes from the forward's offsets and carries no gradient),
//   dx = dr W_r,  dW_r = dr^T x,  db = sum over tokens of dr.
template <typename T>
struct Vec;
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const __nv_bfloat16* p, float* v) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(h[e]);
      v[2 * e] = f.x;
      v[2 * e + 1] = f.y;
    }
  }
  __device__ static void store(__nv_bfloat16* p, const float* v) {
    uint4 u;
    u.x = pack_bf16x2(v[0], v[1]);
    u.y = pack_bf16x2(v[2], v[3]);
    u.z = pack_bf16x2(v[4], v[5]);
    u.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = u;
  }
};
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void load(const float* p, float* v) {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x;
    v[1] = f.y;
    v[2] = f.z;
    v[3] = f.w;
  }
  __device__ static void store(float* p, const float* v) { *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]); }
};

// Router backward from the router's own logits (fp32 [N][M], recomputed by
// the forward router kernels, so they equal the forward's bit for bit).
// dr[i][j] = d(out)/d(r_ij) with p = softmax(r_i) and g = the token's group:
//   dgate_i * p_g * ([j == g] - p_j)  +  bcoef * p_j * (F_j - sum_k F_k p_k)
// (the gate's gradient, and the balancing loss's when bcoef != 0; F_j is the
// share of tokens routed to j).  Written in place over the logits.
__global__ void __launch_bounds__(256)
route_dr_kernel(float* __restrict__ lr, const int32_t* __restrict__ gid, const float* __restrict__ dgate,
                const int32_t* __restrict__ offsets, float bcoef, int64_t N, int M, int* status) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= N) return;
  float* r = lr + i * M;
  const int g = gid[i];
  if (g < 0 || g >= M) {
    if (status) atomicOr(status, DEV_RANGE);
    for (int j = 0; j < M; ++j) r[j] = 0.0f;
    return;
  }
  float mx = -INFINITY;
  for (int j = 0; j < M; ++j) mx = fmaxf(mx, r[j]);
  float z = 0.0f;
  for (int j = 0; j < M; ++j) z += expf(r[j] - mx);
  const float inv = 1.0f / z;
  const float k = dgate[i] * expf(r[g] - mx) * inv;
  float fs = 0.0f;
  const float invN = 1.0f / (float)N;
  if (bcoef != 0.0f)
    for (int j = 0; j < M; ++j) fs += (float)(offsets[j + 1] - offsets[j]) * invN * expf(r[j] - mx) * inv;
  for (int j = 0; j < M; ++j) {
    const float pj = expf(r[j] - mx) * inv;
    float v = k * ((j == g ? 1.0f : 0.0f) - pj);
    if (bcoef != 0.0f) v += bcoef * pj * ((float)(offsets[j + 1] - offsets[j]) * invN - fs);
    r[j] = v;
  }
}

// dx = dr W_r.  A thread owns Vec<T>::n columns and kDxTok tokens per pass,
// so each row of W_r it loads serves kDxTok tokens; dr is read warp-uniformly
// (the same address across the warp).
constexpr int kDxTok = 8;
template <typename T>
__global__ void __launch_bounds__(256)
route_dx_kernel(const T* __restrict__ W, const float* __restrict__ dr, int64_t N, int d, int M, T* __restrict__ dx) {
  constexpr int V = Vec<T>::n;
  const int c = (blockIdx.x * blockDim.x + threadIdx.x) * V;
  if (c >= d) return;  // d is a multiple of V
  for (int64_t t0 = (int64_t)blockIdx.y * kDxTok; t0 < N; t0 += (int64_t)gridDim.y * kDxTok) {
    float acc[kDxTok][V];
#pragma unroll
    for (int tk = 0; tk < kDxTok; ++tk)
#pragma unroll
      for (int e = 0; e < V; ++e) acc[tk][e] = 0.0f;
    const int nt = (int)(N - t0 < kDxTok ? N - t0 : kDxTok);
    for (int j = 0; j < M; ++j) {
      float w[V];
      Vec<T>::load(W + (int64_t)j * d + c, w);
#pragma unroll
      for (int tk = 0; tk < kDxTok; ++tk) {
        const float r = tk < nt ? __ldg(dr + (t0 + tk) * M + j) : 0.0f;
#pragma unroll
        for (int e = 0; e < V; ++e) acc[tk][e] = fmaf(r, w[e], acc[tk][e]);
      }
    }
#pragma unroll
    for (int tk = 0; tk < kDxTok; ++tk)
      if (tk < nt) Vec<T>::store(dx + (t0 + tk) * d + c, acc[tk]);
  }
}

// Partial dW_r = dr^T x and db = sum dr over one slice of the tokens (a
// split-K reduction).  Block (cx, s): each thread owns Vec<T>::n columns of
// x and accumulates them against 16 groups at a time, for the tokens of
// slice s, in chunks of kDwChunk tokens whose dr the block stages in shared
// memory; kDwUnroll rows of x are loaded before they are used, so several
// loads per thread are in flight.  Slices are summed in a fixed order
// afterwards, so the result does not depend on scheduling.
constexpr int kDwGroups = 16;
constexpr int kDwUnroll = 8;
constexpr int kDwThreads = 64;
constexpr int kDwChunk = 64;
template <typename T>
__global__ void __launch_bounds__(kDwThreads)
route_dw_kernel(const T* __restrict__ x, const float* __restrict__ dr, int64_t N, int d, int M, int64_t per_slice,
                float* __restrict__ pw, float* __restrict__ pb) {
  constexpr int V = Vec<T>::n;
  __shared__ float drs[kDwChunk][kDwGroups];
  const int c = (blockIdx.x * kDwThreads + threadIdx.x) * V;
  const int s = blockIdx.y;
  const int64_t i0 = (int64_t)s * per_slice, i1 = min(N, i0 + per_slice);
  const bool col_ok = c < d;  // d is a multiple of V
  const bool bias_lane = blockIdx.x == 0 && threadIdx.x == 0;
  for (int j0 = 0; j0 < M; j0 += kDwGroups) {
    float acc[kDwGroups][V];
    float bacc[kDwGroups];
#pragma unroll
    for (int g = 0; g < kDwGroups; ++g) {
      bacc[g] = 0.0f;
#pragma unroll
      for (int e = 0; e < V; ++e) acc[g][e] = 0.0f;
    }
    for (int64_t cb = i0; cb < i1; cb += kDwChunk) {
      const int nc = (int)(i1 - cb < kDwChunk ? i1 - cb : kDwChunk);
      __syncthreads();  // the previous chunk has been consumed
      for (int e = threadIdx.x; e < kDwChunk * kDwGroups; e += kDwThreads) {
        const int r = e / kDwGroups, g = e - r * kDwGroups;
        drs[r][g] = (r < nc && j0 + g < M) ? dr[(cb + r) * M + j0 + g] : 0.0f;
      }
      __syncthreads();
      for (int u0 = 0; u0 < nc; u0 += kDwUnroll) {
        float xv[kDwUnroll][V];
#pragma unroll
        for (int u = 0; u < kDwUnroll; ++u) {
          if (col_ok && u0 + u < nc)
            Vec<T>::load(x + (cb + u0 + u) * d + c, xv[u]);
          else
#pragma unroll
            for (int e = 0; e < V; ++e) xv[u][e] = 0.0f;
        }
        // rows past the chunk have x = 0 and dr = 0: they add nothing
#pragma unroll
        for (int u = 0; u < kDwUnroll; ++u) {
          const int rr = (u0 + u) < kDwChunk ? u0 + u : kDwChunk - 1;
#pragma unroll
          for (int g = 0; g < kDwGroups; ++g) {
            const float r = (u0 + u) < nc ? drs[rr][g] : 0.0f;
            if (bias_lane) bacc[g] += r;
#pragma unroll
            for (int e = 0; e < V; ++e) acc[g][e] = fmaf(r, xv[u][e], acc[g][e]);
          }
        }
      }
    }
#pragma unroll
    for (int g = 0; g < kDwGroups; ++g) {
      const int j = j0 + g;
      if (j >= M) break;
      if (col_ok) {
        float* dst = pw + ((int64_t)s * M + j) * d + c;
#pragma unroll
        for (int e = 0; e < V; ++e) dst[e] = acc[g][e];
      }
      if (bias_lane) pb[(int64_t)s * M + j] = bacc[g];
    }
  }
}

__global__ void __launch_bounds__(256) route_dw_reduce_kernel(const float* __restrict__ pw,
                                                              const float* __restrict__ pb, int slices, int M, int d,
                                                              float* __restrict__ dW, float* __restrict__ db) {
  const int64_t n = (int64_t)M * d;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int k = 0; k < slices; ++k) s += pw[(int64_t)k * n + e];
    dW[e] = s;
  }
  if (db && blockIdx.x == 0) {
    for (int j = threadIdx.x; j < M; j += blockDim.x) {
      float s = 0.0f;
      for (int k = 0; k < slices; ++k) s += pb[(int64_t)k * M + j];
      db[j] = s;
    }
  }
}

}  // namespace

cudaError_t launch_attn_bwd(const DevCtx& c, const BwdArgs& a, bool dq) {
  if (a.d_h == 128) return dq ? launch_bwd_dh<128, true>(c, a) : launch_bwd_dh<128, false>(c, a);
  if (a.d_h == 64) return dq ? launch_bwd_dh<64, true>(c, a) : launch_bwd_dh<64, false>(c, a);
  return cudaErrorInvalidValue;
}

cudaError_t launch_bwd_prep(const DevCtx& c, const void* dout, const void* o, const int32_t* perm, const float* gate,
                            float w, int64_t N, int H, int d_h, void* dO_hat, float* dsum, float* dgate) {
  if (N == 0) return cudaSuccess;
  int64_t blocks = ceil_div(N, 8);
  const int64_t cap = (int64_t)c.num_sms * 8;
  if (blocks > cap) blocks = cap;
  bwd_prep_kernel<<<(unsigned)blocks, 256, 0, c.stream>>>((const uint4*)dout, (const uint4*)o, perm, gate, w, N, H,
                                                           d_h / 8, (uint4*)dO_hat, dsum, dgate, c.status);
  return cudaGetLastError();
}

cudaError_t launch_mean(const DevCtx& c, const void* x, const void* y, const void* z, int64_t n, void* out) {
  const int64_t n8 = n / 8;
  if (n8 == 0) return cudaSuccess;
  int64_t blocks = ceil_div(n8, 256);
  const int64_t cap = (int64_t)c.num_sms * 8;
  if (blocks > cap) blocks = cap;
  mean_kernel<<<(unsigned)blocks, 256, 0, c.stream>>>((const uint4*)x, (const uint4*)y, (const uint4*)z, n8,
                                                      (uint4*)out);
  return cudaGetLastError();
}

// Token slices of the dW_r partial sums: at most kRouteSlices, and at most
// 64 MiB of partials.
static int route_max_slices(int d, int M) {
  const int64_t per = (int64_t)M * d * 4;
  return (int)std::max<int64_t>(1, std::min<int64_t>(kRouteSlices, ((int64_t)64 << 20) / per));
}

// Workspace of the router backward: the logits (then dr) [N][M], the
// router's group ids, gates and histograms (recomputed, not used), and the
// dW_r / db partial sums.
struct RouteBwdWs {
  size_t lr, gid, gate, hist, pw, pb, total;
};
static RouteBwdWs route_bwd_ws(int64_t N, int d, int M) {
  RouteBwdWs w;
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off += align_up(n, 256);
    return o;
  };
  const size_t S = (size_t)route_max_slices(d, M);
  w.lr = take((size_t)N * M * 4);
  w.gid = take((size_t)N * 4);
  w.gate = take((size_t)N * 4);
  w.hist = take((size_t)ceil_div(N, kTile) * M * 4);
  w.pw = take(S * M * d * 4);
  w.pb = take(S * M * 4);
  w.total = off;
  return w;
}

size_t route_bwd_ws_bytes(int64_t N, int d, int M) { return route_bwd_ws(N, d, M).total; }

cudaError_t launch_route_bwd(const DevCtx& c, const void* x, const void* W, const float* b, bool bf16, int64_t N,
                             int d, int M, const int32_t* gid, const float* dgate, const int32_t* offsets,
                             float balance_alpha, void* dx, float* dW, float* db, uint8_t* ws) {
  const float bcoef = N > 0 ? balance_alpha * (float)M / (float)N : 0.0f;
  const RouteBwdWs w = route_bwd_ws(N, d, M);
  float* lr = reinterpret_cast<float*>(ws + w.lr);
  float* pw = reinterpret_cast<float*>(ws + w.pw);
  float* pb = reinterpret_cast<float*>(ws + w.pb);
  cudaError_t e;
  if (N > 0) {
    // the logits, from the same router kernel the forward used
    int32_t* gid2 = reinterpret_cast<int32_t*>(ws + w.gid);
    float* gate2 = reinterpret_cast<float*>(ws + w.gate);
    int32_t* hist = reinterpret_cast<int32_t*>(ws + w.hist);
    if (bf16 && M <= 256 && d >= 64)
      e = launch_route_tc(c, x, W, b, N, d, M, gid2, gate2, hist, nullptr, lr);
    else
      e = launch_route_simt(c, x, W, b, bf16, N, d, M, gid2, gate2, hist, nullptr, lr);
    if (e != cudaSuccess) return e;
    route_dr_kernel<<<(unsigned)ceil_div(N, 256), 256, 0, c.stream>>>(lr, gid, dgate, offsets, bcoef, N, M,
                                                                       c.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int vec = bf16 ? 8 : 4;
    const int64_t lanes = ceil_div(d, vec);
    const int threads = (int)std::min<int64_t>(256, ceil_div(lanes, 32) * 32);
    const int64_t cxb = ceil_div(lanes, threads);
    const int64_t ty = std::max<int64_t>(1, std::min<int64_t>(ceil_div(N, kDxTok), (int64_t)c.num_sms * 8 / cxb));
    dim3 grid((unsigned)cxb, (unsigned)ty);
    if (bf16)
      route_dx_kernel<__nv_bfloat16><<<grid, threads, 0, c.stream>>>((const __nv_bfloat16*)W, lr, N, d, M,
                                                                      (__nv_bfloat16*)dx);
    else
      route_dx_kernel<float><<<grid, threads, 0, c.stream>>>((const float*)W, lr, N, d, M, (float*)dx);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // enough blocks of kDwThreads to keep x's reads in flight: column blocks
  // times token slices, about eight blocks per SM
  const int vec = bf16 ? 8 : 4;
  const int64_t cx = ceil_div(ceil_div(d, vec), kDwThreads);
  const int slices = (int)std::min<int64_t>(route_max_slices(d, M), std::max<int64_t>(1, 8 * c.num_sms / cx));
  const int64_t per = ceil_div(N > 0 ? N : 1, slices);
  dim3 grid((unsigned)cx, (unsigned)slices);
  if (bf16)
    route_dw_kernel<__nv_bfloat16><<<grid, kDwThreads, 0, c.stream>>>((const __nv_bfloat16*)x, lr, N, d, M, per, pw,
                                                                       pb);
  else
    route_dw_kernel<float><<<grid, kDwThreads, 0, c.stream>>>((const float*)x, lr, N, d, M, per, pw, pb);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  int64_t blocks = ceil_div((int64_t)M * d, 256);
  if (blocks > 1024) blocks = 1024;
  route_dw_reduce_kernel<<<(unsigned)blocks, 256, 0, c.stream>>>(pw, pb, slices, M, d, dW, db);
  return cudaGetLastError();
}

}  // namespace moga
