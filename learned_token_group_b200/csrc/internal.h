// Internal launchers shared by the kernel files and the C ABI (api.cu).
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace moga {

constexpr int kTile = 128;  // tokens per routing tile / query rows per attention tile

// Device status bits, OR-ed into the workspace status word.
enum : int {
  DEV_TIMEOUT = 1,  // an mbarrier wait ran past its limit
  DEV_RANGE = 2,    // an index or offsets array was out of range (the access was skipped)
};

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct DevCtx {
  cudaStream_t stream;
  int* status;        // device status word (workspace header)
  uint64_t wait_ns;   // bound on any single device-side wait
  int num_sms;
  int device;
};

// ------------------------------------------------------------------ routing
// Router logits + softmax gate + argmax + per-tile group histogram.
// pstat (nullable): per (tile, warp) sums of p(i|x) over the warp's tokens, [tiles][4][M].
cudaError_t launch_route_tc(const DevCtx& c, const void* x, const void* W, const float* b, int64_t N, int d,
                            int M, int32_t* group_id, float* gate, int32_t* hist, float* pstat);
cudaError_t launch_route_simt(const DevCtx& c, const void* x, const void* W, const float* b, bool bf16,
                              int64_t N, int d, int M, int32_t* group_id, float* gate, int32_t* hist, float* pstat);
// Exclusive scan of the per-tile histograms -> offsets, max_seqlen, per-tile
// bases; with pstat also the mean routing probabilities and the balance metric.
cudaError_t launch_scan(const DevCtx& c, const int32_t* hist, int64_t ntiles, int M, int32_t* base,
                        int32_t* offsets, int32_t* max_seqlen, const float* pstat, int64_t N, float* prob_mean,
                        float* balance);
// Stable scatter of token indices into perm.
cudaError_t launch_scatter(const DevCtx& c, const int32_t* group_id, const int32_t* base, int64_t N, int M,
                           int32_t* perm);

// ------------------------------------------------------------------ attention
// Window-order permutation of the STGA grid.
cudaError_t launch_window_perm(const DevCtx& c, int T, int Hg, int Wg, const int* window, int32_t* perm_w);
// Sorted segment table (largest group first) for the grouped attention.
cudaError_t launch_seg_table(const DevCtx& c, const int32_t* offsets, int M, int H, int64_t N, int32_t* table);

// Q/K/V rows gathered by perm into head-major [H][N][d_h] buffers.
cudaError_t launch_gather(const DevCtx& c, const void* q, const void* k, const void* v, const int32_t* perm,
                          int64_t N, int H, int d_h, void* qh, void* kh, void* vh);

struct AttnArgs {
  // direct = 1: q, k, v are the caller's [N, H, d_h] tensors, read by token
  // index (perm); direct = 0: they are gathered head-major copies [H][N][d_h].
  int direct;
  const void* q;
  const void* k;
  const void* v;
  const int32_t* perm;    // segment position -> original token
  const float* gate;      // per original token, or null (gate = 1)
  void* out;              // bf16 [N, H, d_h]
  int64_t N;
  int H;
  int d_h;
  float out_scale;
  int accumulate;         // 0: out = scale*gate*O ; 1: out += scale*O
  // segment source: groups (sorted table in device memory) or STGA windows
  int mode;               // 0 groups, 1 windows
  const int32_t* table;   // groups: [3*(M+1)] = tile_prefix | seg_start | seg_len (sorted)
  int nseg;               // groups: M ; windows: number of windows
  int T, Hg, Wg, wt, wh, ww;
  int debug_withhold_first_k;  // test hook: the producer skips each CTA's first K tile
};
cudaError_t launch_attention(const DevCtx& c, const AttnArgs& a);

// Number of STGA windows for a grid.
inline int64_t stga_num_windows(int T, int Hg, int Wg, const int* w) {
  return ceil_div(T, w[0]) * ceil_div(Hg, w[1]) * ceil_div(Wg, w[2]);
}

// Encodes a 2-D bf16 tensor map (inner dim contiguous) with a 64 x box_rows
// box and 128-byte swizzle.  Returns false if the driver entry point is
// unavailable or the encoding fails.
bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                  uint32_t box_rows);

}  // namespace moga
