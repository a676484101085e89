// STGA window attention for windows of up to 192 tokens ("MoGA: Mixture-of-Groups Attention
// for End-to-End Long Video Generation", §3.4 "Spatial-Temporal Group
// Attention (STGA)"): full softmax attention inside every non-overlapping
// (wt, wh, ww) box of the (T, Hg, Wg) latent grid, boxes anchored at the
// origin and clipped at the grid's edges.
//
// stga_kernel<DH, NSC>  persistent, one CTA per SM, one (window, head) per
//   step.  Every window, clipped or not, is loaded as one 5-D TMA box per
//   64-column chunk: the tensor map views q, k, v [T*Hg*Wg, H, d_h] as
//   (d_h, H, Wg, Hg, T), and a box of (64, 1, ww, wh, wt) lands as wt*wh*ww
//   rows of 128 bytes in box order, row = (f*wh + i)*ww + j.  Coordinates
//   past the grid's edge are filled with zeros, so a clipped window is a box
//   with zero rows: those keys are masked and those queries dropped.
//
//   S = Q K^T covers all keys of the box in one N <= 192 product, so the
//   softmax needs no online rescaling.  Query tile A is box rows 0-127; tile
//   B starts at box row 64, so its live rows (128-191) sit in TMEM lanes
//   64-127, which warps 2 and 3 can read: 256 threads hold the CTA.
//     warp 0      TMA producer: per step the V tile into one of two slots,
//                 then Q and K into the single Q/K stage
//     warp 1      TMEM allocation; one lane issues tcgen05.mma
//     warps 2-3   softmax + epilogue of tile B (box rows 128-191)
//     warps 4-7   softmax + epilogue of tile A (box rows 0-127)
//   TMEM (512 columns): tile A S [0, 192), P (bf16 pairs) over [0, 96),
//   O [128, 128 + d_h); tile B the same from column 256.  O overlaps the top
//   of S: the P V product that writes O is issued only after the softmax has
//   read all of S, and the next step's S waits until the epilogue has read O.
//   Every wait is bounded (status word + abort flag, as in attn.cu).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"
#include "windows.cuh"

namespace moga {

namespace {

constexpr int kStgaThreads = 256;
constexpr int kBoxRowsMax = 192;               // largest window box (tokens)
constexpr int kStgaChunk = kBoxRowsMax * 128;  // one 64-column chunk of a window tile: 24 KB

template <int DH>
struct StgaPlan {
  static constexpr int kChunks = DH / 64;
  static constexpr int kTileBytes = kChunks * kStgaChunk;  // Q, K or V of one window and head
  static constexpr int kQ = 0;
  static constexpr int kK = kTileBytes;
  static constexpr int kV0 = 2 * kTileBytes;  // [2] V slots
  static constexpr int kBar = 4 * kTileBytes;
  static constexpr size_t kBytes = (size_t)kBar + 256 + 1024;  // barriers + alignment slack
};

struct StgaArgs {
  void* out;         // bf16 [N, H, d_h]
  float* lse;        // nullable: [H][N] natural-log log-sum-exp at window-order positions
  int64_t N;
  int H;
  int T, Hg, Wg, wt, wh, ww, nbh, nbw;
  int nwin;          // number of windows
  int box;           // wt * wh * ww (<= 192)
  float out_scale;
  int accumulate;    // 0: out = scale * O / l ; 1: out += scale * O / l
  int withhold;      // test hook: the first Q/K load is never issued
};

__device__ __forceinline__ void tma_load_5d(const CUtensorMap* map, uint64_t* bar, void* dst, int c0, int c1,
                                            int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// Window seg -> its origin (t0, h0, w0) and clipped extents (et, eh, ew).
struct WinBox {
  int t0, h0, w0, et, eh, ew;
};
__device__ __forceinline__ WinBox win_box(const StgaArgs& a, int seg) {
  WinBox b;
  const int tb = seg / (a.nbh * a.nbw);
  const int hb = (seg / a.nbw) % a.nbh;
  const int wb = seg % a.nbw;
  b.t0 = tb * a.wt;
  b.h0 = hb * a.wh;
  b.w0 = wb * a.ww;
  b.et = min(a.wt, a.T - b.t0);
  b.eh = min(a.wh, a.Hg - b.h0);
  b.ew = min(a.ww, a.Wg - b.w0);
  return b;
}

// NSC: 32-column chunks of S the softmax reads (keys rounded up to 32).
template <int DH, int NSC>
__global__ void __launch_bounds__(kStgaThreads, 1)
stga_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
            const __grid_constant__ CUtensorMap tv, const StgaArgs a, int* status, unsigned long long wait_ns) {
  using P = StgaPlan<DH>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::kBar);
  uint64_t* qk_full = bars + 0;
  uint64_t* qk_empty = bars + 1;
  uint64_t* v_full = bars + 2;   // [2]
  uint64_t* v_empty = bars + 4;  // [2]
  uint64_t* s_full = bars + 6;   // [2] S of tile A / B computed
  uint64_t* p_full = bars + 8;   // [2] P of tile A / B written
  uint64_t* o_full = bars + 10;  // [2] P V of tile A / B done
  uint64_t* o_free = bars + 12;  // [2] O of tile A / B read by the epilogue
  uint64_t* done_bar = bars + 14;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 15);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int B = a.box;
  const bool has_b = B > kTile;  // a second query tile (box rows 128..B-1)
  // threads of each tile whose warp holds at least one box row < B
  const int cnt_a = 32 * ((min(B, kTile) + 31) / 32);
  const int cnt_b = has_b ? 32 * ((B - kTile + 31) / 32) : 0;

  if (threadIdx.x == 0) {
    mbar_init(qk_full, 1);
    mbar_init(qk_empty, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&o_full[s], 1);
    }
    mbar_init(&p_full[0], cnt_a);
    mbar_init(&o_free[0], cnt_a);
    mbar_init(&p_full[1], cnt_b > 0 ? cnt_b : 1);
    mbar_init(&o_free[1], cnt_b > 0 ? cnt_b : 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  {
    // Rows past a box (B .. 191) are never written by TMA; they start as
    // zeros, so every operand row the tensor core reads is finite.
    uint4* t = reinterpret_cast<uint4*>(smem);
    for (int i = threadIdx.x; i < P::kBar / 16; i += kStgaThreads) t[i] = make_uint4(0, 0, 0, 0);
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto tS = [tmem](int x) { return tmem + (uint32_t)(x * 256); };
  auto tO = [tmem](int x) { return tmem + (uint32_t)(x * 256 + 128); };
  WaitCtx wc{abort_flag, status, wait_ns};
  const int H = a.H;
  const int total = a.nwin * H;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      const uint32_t box_bytes = (uint32_t)B * 128u;  // one 64-column chunk of one tensor
      int last_qk = -1;
      int last_v[2] = {-1, -1};
      uint32_t i = 0;
      for (int idx = blockIdx.x; idx < total; idx += gridDim.x, ++i) {
        const int h = idx % H;
        const WinBox w = win_box(a, idx / H);
        const int s = (int)(i & 1);
        const uint32_t u = i >> 1;
        // V first: its slot frees earlier (after the P V product two steps
        // back) than the Q/K stage (after the previous step's S products).
        if (!mbar_wait(&v_empty[s], (u & 1) ^ 1, wc, 3, i)) break;
        mbar_expect_tx(&v_full[s], (uint32_t)P::kChunks * box_bytes);
#pragma unroll
        for (int c = 0; c < P::kChunks; ++c)
          tma_load_5d(&tv, &v_full[s], smem + P::kV0 + s * P::kTileBytes + c * kStgaChunk, c * 64, h, w.w0, w.h0,
                      w.t0);
        last_v[s] = (int)u;
        if (!mbar_wait(qk_empty, (i & 1) ^ 1, wc, 1, i)) break;
        // Test hook: this Q/K load never arrives, so the MMA warp's bounded
        // wait runs out and the kernel reports a timeout.
        if (a.withhold && i == 0) break;
        mbar_expect_tx(qk_full, 2u * (uint32_t)P::kChunks * box_bytes);
#pragma unroll
        for (int c = 0; c < P::kChunks; ++c) {
          tma_load_5d(&tq, qk_full, smem + P::kQ + c * kStgaChunk, c * 64, h, w.w0, w.h0, w.t0);
          tma_load_5d(&tk, qk_full, smem + P::kK + c * kStgaChunk, c * 64, h, w.w0, w.h0, w.t0);
        }
        last_qk = (int)i;
      }
      // Drain every load this thread issued before the CTA exits.
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      if (last_qk >= 0) mbar_wait(qk_full, (uint32_t)last_qk & 1, dc);
      for (int s = 0; s < 2; ++s)
        if (last_v[s] >= 0) mbar_wait(&v_full[s], (uint32_t)last_v[s] & 1, dc);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const int ns = (B + 15) & ~15;  // keys of the S product (N)
      const uint32_t idS = idesc_bf16(128, ns, false, false);
      constexpr uint32_t idO = idesc_bf16(128, DH, false, true);
      const uint32_t qa = smem_u32(smem + P::kQ);
      const uint64_t qd[2] = {sdesc_sw128(qa, 16, 1024), sdesc_sw128(qa + 64 * 128, 16, 1024)};
      const uint64_t kd = sdesc_sw128(smem_u32(smem + P::kK), 16, 1024);
      const uint64_t vd[2] = {sdesc_sw128(smem_u32(smem + P::kV0), kStgaChunk, 1024),
                              sdesc_sw128(smem_u32(smem + P::kV0 + P::kTileBytes), kStgaChunk, 1024)};
      const int nkk = ns / 16;
      // S_x = Q_x K^T: tile A reads box rows 0-127, tile B rows 64-191.
      auto issue_s = [&](int x) {
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (uint32_t)((kk >> 2) * kStgaChunk + (kk & 3) * 32);
          umma_bf16(tS(x), sdesc_add(qd[x], off), sdesc_add(kd, off), idS, kk > 0 ? 1u : 0u);
        }
      };
      // O_x = P_x V, P from TMEM over S_x, V MN-major (chunks kStgaChunk apart).
      auto issue_pv = [&](int x, int s) {
        for (int kk = 0; kk < nkk; ++kk)
          umma_bf16_ts(tO(x), tS(x) + kk * 8, sdesc_add(vd[s], kk * 2048), idO, kk > 0 ? 1u : 0u);
      };
      uint32_t i = 0;
      for (int idx = blockIdx.x; idx < total; idx += gridDim.x, ++i) {
        if (!mbar_wait(qk_full, i & 1, wc, 4, i)) break;
        // S_x overwrites the columns of the previous step's O_x: wait until
        // the epilogue has read them.
        if (i > 0 && !mbar_wait(&o_free[0], (i - 1) & 1, wc, 10, i)) break;
        tc_fence_after();
        issue_s(0);
        umma_commit(&s_full[0]);
        if (has_b) {
          if (i > 0 && !mbar_wait(&o_free[1], (i - 1) & 1, wc, 26, i)) break;
          tc_fence_after();
          issue_s(1);
          umma_commit(&s_full[1]);
        }
        umma_commit(qk_empty);
        const int s = (int)(i & 1);
        if (!mbar_wait(&v_full[s], (i >> 1) & 1, wc, 7, i)) break;
        if (!mbar_wait(&p_full[0], i & 1, wc, 13, i)) break;
        tc_fence_after();
        issue_pv(0, s);
        umma_commit(&o_full[0]);
        if (has_b) {
          if (!mbar_wait(&p_full[1], i & 1, wc, 29, i)) break;
          tc_fence_after();
          issue_pv(1, s);
          umma_commit(&o_full[1]);
        }
        umma_commit(&v_empty[s]);
      }
      umma_commit(done_bar);
      volatile int zero = 0;
      WaitCtx dc{&zero, nullptr, 100000000ull};
      mbar_wait(done_bar, 0, dc);
    }
  } else {
    // ---------------------------------------------------------------- softmax + epilogue
    const bool tile_b = warp < 4;  // warps 2-3: tile B; warps 4-7: tile A
    const int x = tile_b ? 1 : 0;
    const int sub = warp & 3;       // TMEM sub-partition this warp may access
    const int lr = sub * 32 + lane; // TMEM lane
    const int r = tile_b ? 64 + lr : lr;  // this thread's box row (query)
    const int r0 = r - lane;              // the warp's first box row
    const bool live_warp = tile_b ? (has_b && r0 < B) : (r0 < B);
    if (live_warp) {
      const uint32_t lane_base = (uint32_t)(sub * 32) << 16;
      const uint32_t tSx = tS(x) + lane_base, tOx = tO(x) + lane_base;
      const float scale_log2 = 1.4426950408889634f * rsqrtf((float)DH);
      const int plane = a.wh * a.ww;
      // box coordinates of this thread's query row and of the key column this
      // lane stands for in each 32-column word of the mask
      const int rf = r / plane, ri = (r / a.ww) % a.wh, rj = r % a.ww;
      // (frame << 16 | row << 8 | column) of the key column; window extents
      // are at most 256, so each field fits, and columns past the box get a
      // frame no window reaches
      uint32_t ck[NSC];
#pragma unroll
      for (int w = 0; w < NSC; ++w) {
        const int c = 32 * w + lane;
        const uint32_t f = c < B ? (uint32_t)(c / plane) : 0x7fffu;
        ck[w] = (f << 16) | ((uint32_t)((c / a.ww) % a.wh) << 8) | (uint32_t)(c % a.ww);
      }
      uint32_t i = 0;
      for (int idx = blockIdx.x; idx < total; idx += gridDim.x, ++i) {
        const int h = idx % H;
        const int seg = idx / H;
        const WinBox w = win_box(a, seg);
        const bool row_ok = r < B && rf < w.et && ri < w.eh && rj < w.ew;
        const int64_t tok = ((int64_t)(w.t0 + rf) * a.Hg + (w.h0 + ri)) * a.Wg + (w.w0 + rj);
        // valid keys of this window, one bit per box row
        uint32_t mw[NSC];
        bool all_valid = true;
#pragma unroll
        for (int ww = 0; ww < NSC; ++ww) {
          const uint32_t k = ck[ww];
          mw[ww] = __ballot_sync(0xffffffffu, (int)(k >> 16) < w.et && (int)((k >> 8) & 0xffu) < w.eh &&
                                                  (int)(k & 0xffu) < w.ew);
          all_valid = all_valid && mw[ww] == 0xffffffffu;
        }
        if (!mbar_wait(&s_full[x], i & 1, wc, 6 + 16 * x, i)) break;
        tc_fence_after();
        float sr[NSC * 32];
#pragma unroll
        for (int c = 0; c < NSC; ++c) tmem_ld32(tSx + c * 32, sr + c * 32);
        tmem_ld_wait();
        if (!all_valid) {
#pragma unroll
          for (int c = 0; c < NSC * 32; ++c)
            if (!((mw[c >> 5] >> (c & 31)) & 1u)) sr[c] = -INFINITY;
        }
        // row max: independent chains of 3-input maxima
        float m8[NSC * 2];
#pragma unroll
        for (int g = 0; g < NSC * 2; ++g) {
          float m = fmax3(sr[16 * g], sr[16 * g + 1], sr[16 * g + 2]);
#pragma unroll
          for (int k = 3; k + 1 < 16; k += 2) m = fmax3(m, sr[16 * g + k], sr[16 * g + k + 1]);
          m8[g] = fmaxf(m, sr[16 * g + 15]);
        }
        float mx = m8[0];
#pragma unroll
        for (int g = 1; g < NSC * 2; ++g) mx = fmaxf(mx, m8[g]);
        const float m = mx * scale_log2;
        // P = 2^(S*scale - m) as packed bf16 pairs over S; l = sum of P
        const uint64_t sc2 = f2_pack(scale_log2, scale_log2);
        const uint64_t nm2 = f2_pack(-m, -m);
        uint64_t la = f2_pack(0.f, 0.f), lb = la;
#pragma unroll
        for (int c = 0; c < NSC; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint64_t t2 = f2_fma(f2_pack(sr[c * 32 + 2 * e], sr[c * 32 + 2 * e + 1]), sc2, nm2);
            float t0, t1;
            f2_unpack(t2, t0, t1);
            const float p0 = fast_exp2(t0), p1 = fast_exp2(t1);
            if (e & 1)
              lb = f2_add(lb, f2_pack(p0, p1));
            else
              la = f2_add(la, f2_pack(p0, p1));
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st16u(tSx + c * 16, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[x]);
        // epilogue: read O, release its columns, then normalise and write
        if (!mbar_wait(&o_full[x], i & 1, wc, 9 + 16 * x, i)) break;
        tc_fence_after();
        float o[DH];
#pragma unroll
        for (int c = 0; c < DH / 32; ++c) tmem_ld32(tOx + c * 32, o + c * 32);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&o_free[x]);
        float l0, l1;
        f2_unpack(f2_add(la, lb), l0, l1);
        const float l = l0 + l1;
        if (row_ok && h < H && tok < a.N) {
          if (a.lse) {
            // window-order position of the token: the window's start plus
            // its row-major index inside the clipped window
            const int start = w.t0 * a.Hg * a.Wg + w.et * (w.h0 * a.Wg + w.eh * w.w0);
            const int pos = start + (rf * w.eh + ri) * w.ew + rj;
            a.lse[(int64_t)h * a.N + pos] = (m + log2f(l)) * 0.6931471805599453f;
          }
          const float inv = a.out_scale / l;
          uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                                (tok * H + h) * (int64_t)DH);
#pragma unroll
          for (int q4 = 0; q4 < DH / 8; ++q4) {
            uint4 pk;
            pk.x = pack_bf16x2(o[q4 * 8 + 0] * inv, o[q4 * 8 + 1] * inv);
            pk.y = pack_bf16x2(o[q4 * 8 + 2] * inv, o[q4 * 8 + 3] * inv);
            pk.z = pack_bf16x2(o[q4 * 8 + 4] * inv, o[q4 * 8 + 5] * inv);
            pk.w = pack_bf16x2(o[q4 * 8 + 6] * inv, o[q4 * 8 + 7] * inv);
            if (a.accumulate)
              red_add_bf16x8(dst + q4, pk);
            else
              dst[q4] = pk;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DH, int NSC>
cudaError_t launch_nsc(const DevCtx& c, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                       const StgaArgs& s, int grid) {
  auto kern = stga_kernel<DH, NSC>;
  const size_t smem = StgaPlan<DH>::kBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, kStgaThreads, smem, c.stream>>>(mq, mk, mv, s, c.status, (unsigned long long)c.wait_ns);
  return cudaGetLastError();
}

template <int DH>
cudaError_t launch_dh(const DevCtx& c, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                      const StgaArgs& s, int grid) {
  if (s.box <= 64) return launch_nsc<DH, 2>(c, mq, mk, mv, s, grid);
  if (s.box <= 128) return launch_nsc<DH, 4>(c, mq, mk, mv, s, grid);
  return launch_nsc<DH, 6>(c, mq, mk, mv, s, grid);
}

}  // namespace

bool stga_box_supported(int d_h, const int* window) {
  if (d_h != 64 && d_h != 128) return false;
  if (window[0] < 1 || window[1] < 1 || window[2] < 1) return false;
  return (int64_t)window[0] * window[1] * window[2] <= kBoxRowsMax;
}

cudaError_t launch_stga_box(const DevCtx& c, const AttnArgs& a, bool* handled) {
  *handled = false;
  const int win[3] = {a.wt, a.wh, a.ww};
  if (a.mode != 1 || !stga_box_supported(a.d_h, win) || a.gate) return cudaSuccess;
  CUtensorMap mq, mk, mv;
  if (!make_tmap_box5(&mq, a.q, a.d_h, a.H, a.Wg, a.Hg, a.T, win) ||
      !make_tmap_box5(&mk, a.k, a.d_h, a.H, a.Wg, a.Hg, a.T, win) ||
      !make_tmap_box5(&mv, a.v, a.d_h, a.H, a.Wg, a.Hg, a.T, win))
    return cudaSuccess;  // not encodable: the caller keeps the general kernel
  *handled = true;
  StgaArgs s{};
  s.out = a.out;
  s.lse = a.lse;
  s.N = a.N;
  s.H = a.H;
  s.T = a.T;
  s.Hg = a.Hg;
  s.Wg = a.Wg;
  s.wt = a.wt;
  s.wh = a.wh;
  s.ww = a.ww;
  s.nbh = (int)ceil_div(a.Hg, a.wh);
  s.nbw = (int)ceil_div(a.Wg, a.ww);
  s.nwin = a.nseg;
  s.box = a.wt * a.wh * a.ww;
  s.out_scale = a.out_scale;
  s.accumulate = a.accumulate;
  s.withhold = a.debug_withhold_first_k;
  const int64_t total = (int64_t)s.nwin * s.H;
  if (total == 0) return cudaSuccess;
  const int grid = (int)(total < c.num_sms ? total : c.num_sms);
  return a.d_h == 128 ? launch_dh<128>(c, mq, mk, mv, s, grid) : launch_dh<64>(c, mq, mk, mv, s, grid);
}

}  // namespace moga
