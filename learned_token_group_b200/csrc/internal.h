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
// logits (nullable): the logits x W_r^T + b_r themselves, fp32 [N][M].
cudaError_t launch_route_tc(const DevCtx& c, const void* x, const void* W, const float* b, int64_t N, int d,
                            int M, int32_t* group_id, float* gate, int32_t* hist, float* pstat,
                            float* logits = nullptr);
cudaError_t launch_route_simt(const DevCtx& c, const void* x, const void* W, const float* b, bool bf16,
                              int64_t N, int d, int M, int32_t* group_id, float* gate, int32_t* hist, float* pstat,
                              float* logits = nullptr);
// Exclusive scan of the per-tile histograms -> offsets, max_seqlen, per-tile
// bases; with pstat also the mean routing probabilities and the balance metric.
cudaError_t launch_scan(const DevCtx& c, const int32_t* hist, int64_t ntiles, int M, int32_t* base,
                        int32_t* offsets, int32_t* max_seqlen, const float* pstat, int64_t N, float* prob_mean,
                        float* balance);
// Per-tile group histograms of caller-given group ids (ids outside [0, M)
// are skipped and reported as DEV_RANGE).
cudaError_t launch_hist(const DevCtx& c, const int32_t* group_id, int64_t N, int M, int32_t* hist);
// Stable scatter of token indices into perm (ids outside [0, M) are skipped).
cudaError_t launch_scatter(const DevCtx& c, const int32_t* group_id, const int32_t* base, int64_t N, int M,
                           int32_t* perm);

// ------------------------------------------------------------------ attention
// Window-order permutation of the STGA grid.
cudaError_t launch_window_perm(const DevCtx& c, int T, int Hg, int Wg, const int* window, int32_t* perm_w);
// Sorted segment table (largest group first) for the grouped attention; a
// work unit is tiles_per_unit 128-row tiles of one (group, head).
cudaError_t launch_seg_table(const DevCtx& c, const int32_t* offsets, int M, int H, int64_t N, int32_t* table,
                             int tiles_per_unit = 2);

// Q/K/V rows gathered by perm into head-major [H][N][d_h] buffers.
cudaError_t launch_gather(const DevCtx& c, const void* q, const void* k, const void* v, const int32_t* perm,
                          int64_t N, int H, int d_h, void* qh, void* kh, void* vh);

// Rows idx[0..rows) of a (and b) gathered head-major into da (db) with a
// per-head row stride; rows = *rows_dev when given, else rows_max.
cudaError_t launch_gather_rows(const DevCtx& c, const void* a, const void* b, const int32_t* idx,
                               const int32_t* rows_dev, int64_t rows_max, int64_t N, int H, int d_h, int64_t stride,
                               void* da, void* db);

struct AttnArgs {
  // direct = 1: q, k, v are the caller's [N, H, d_h] tensors, read by token
  // index (perm); direct = 0: they are gathered head-major copies [H][N][d_h].
  int direct;
  // contiguous = 1 (tiled kernel): segments are runs of consecutive tokens
  // (windows of whole frames), so q, k, v are the caller's [N, H, d_h]
  // tensors read in place with 3-D maps and perm is the identity (may be null).
  int contiguous;
  const void* q;
  const void* k;
  const void* v;
  const int32_t* perm;    // segment position -> original token (queries; also keys/values unless kvperm)
  const int32_t* kvperm;  // mode 2: key/value position -> original token
  const float* gate;      // per original token, or null (gate = 1)
  void* out;              // bf16 [N, H, d_h]
  int64_t N;
  int64_t kv_rows;        // tiled mode 2: per-head rows of the K/V copies (0: N)
  int H;
  int d_h;
  float out_scale;
  int accumulate;         // 0: out = scale*gate*O ; 1: out += scale*O
  // segment source: groups (sorted table in device memory), STGA windows
  // (decoded from the grid), or shot windows (mode 2: a window table in
  // device memory whose key/value segments differ from the query segments;
  // read in place only)
  int mode;               // 0 groups, 1 windows, 2 shot windows
  const int32_t* table;   // groups: [3*(M+1)] = tile_prefix | seg_start | seg_len (sorted); mode 2: window table
  int nseg;               // groups: M ; windows: number of windows ; mode 2: table capacity (windows)
  int T, Hg, Wg, wt, wh, ww;
  int debug_withhold_first_k;  // test hook: the producer skips each CTA's first K tile
  // modes 0 and 1 (nullable): natural-log log-sum-exp of each query row's
  // scaled scores, [H][N] fp32 at segment positions (the training forward
  // keeps it for the backward pass)
  float* lse;
};
cudaError_t launch_attention(const DevCtx& c, const AttnArgs& a);
// STGA windows of at most 192 tokens (d_h 64 or 128), every window loaded as
// one 5-D TMA box per 64-column chunk (stga.cu).  *handled = false when the
// arguments do not fit it (the caller then runs launch_attention).
bool stga_box_supported(int d_h, const int* window);
cudaError_t launch_stga_box(const DevCtx& c, const AttnArgs& a, bool* handled);

// ------------------------------------------------------------------ training (bwd.cu)
// Attention backward over groups (mode 0) or STGA windows (mode 1).  q, k, v
// and dout are head-major copies [H][N][d_h] in segment order; lse and dsum
// are [H][N] fp32 at segment positions (lse: natural-log log-sum-exp of the
// scaled scores from the forward; dsum: D = sum_c dO*O).  perm maps a
// segment position to its token (null: identity).
struct BwdArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* dout;
  const float* lse;
  const float* dsum;
  const int32_t* perm;
  void* out1;  // dV (dK/dV pass) or dQ (dQ pass): bf16 [N, H, d_h] by token
  void* out2;  // dK (dK/dV pass)
  int64_t N;
  int H;
  int d_h;
  int accumulate;  // 0: store; 1: add into the outputs
  int mode;
  const int32_t* table;  // groups: the segment table with one 128-row tile per unit
  int nseg;
  int T, Hg, Wg, wt, wh, ww;
};
// dq = false: dK and dV (keys stationary); dq = true: dQ (queries stationary).
cudaError_t launch_attn_bwd(const DevCtx& c, const BwdArgs& a, bool dq);
// dO_hat = w * gate * dout gathered by perm (head-major), D, and (when dgate
// is given) the gate gradient sum_h D / gate per token.
cudaError_t launch_bwd_prep(const DevCtx& c, const void* dout, const void* o, const int32_t* perm, const float* gate,
                            float w, int64_t N, int H, int d_h, void* dO_hat, float* dsum, float* dgate);
// out = (x + y + z) / 3, or (x + y) / 2 when z is null, over n bf16 values (n a multiple of 8).
cudaError_t launch_mean(const DevCtx& c, const void* x, const void* y, const void* z, int64_t n, void* out);
// Router backward through the gate (plus, when balance_alpha != 0, the group
// balancing loss alpha * M * sum_i F_i P_i with F from offsets): dx (dtype of
// x), dW_r fp32 [M, d], db fp32 [M] (nullable).
constexpr int kRouteSlices = 512;  // upper bound on token slices of the dW_r partial sums
size_t route_bwd_ws_bytes(int64_t N, int d, int M);
cudaError_t launch_route_bwd(const DevCtx& c, const void* x, const void* W, const float* b, bool bf16, int64_t N,
                             int d, int M, const int32_t* gid, const float* dgate, const int32_t* offsets,
                             float balance_alpha, void* dx, float* dW, float* db, uint8_t* ws);

// ------------------------------------------------------------------ shot windows
// Window table of shot-aware STGA (int32, device):
//   [0] windows, [1] work units (query-tile pairs x heads), [2] key/value rows, [3] spare,
//   [4, 4 + cap + 1)   unit prefix per window,
//   then cap entries of kShotEnt ints: q_start, q_len, kv_start, kv_len,
//   t0, t1 (own frames), pf0, pf1 (previous shot's frames), nf0, nf1 (next
//   shot's frames), tile row, tile column.
constexpr int kShotHdr = 4;
constexpr int kShotEnt = 12;
inline size_t shot_table_ints(int64_t cap) { return (size_t)(kShotHdr + cap + 1 + kShotEnt * cap); }
// Upper bound on the number of windows of any shot split of T frames into nshots shots.
inline int64_t shot_window_cap(int T, int Hg, int Wg, const int* w, int nshots) {
  const int64_t tw = w[0] > 0 ? ((int64_t)T + (int64_t)nshots * (w[0] - 1)) / w[0] : nshots;
  return tw * ceil_div(Hg, w[1]) * ceil_div(Wg, w[2]);
}
// Upper bound on key/value rows: every token once plus the boundary frames of each cut.
inline int64_t shot_kv_cap(int T, int Hg, int Wg, int nshots, int aug_prev, int aug_next) {
  return (int64_t)T * Hg * Wg + (int64_t)(nshots - 1) * (aug_prev + aug_next) * Hg * Wg;
}
// Builds the window table from the device shot boundaries (checked on the device).
cudaError_t launch_shot_table(const DevCtx& c, const int32_t* shot_start, int nshots, int T, int Hg, int Wg,
                              const int* window, int aug_prev, int aug_next, int H, int64_t cap, int32_t* wtab);
// Query and key/value index lists of every window of the table.
cudaError_t launch_shot_perm(const DevCtx& c, const int32_t* wtab, int64_t cap, int Hg, int Wg, const int* window,
                             int32_t* qperm, int32_t* kvperm);

// Number of STGA windows for a grid.
inline int64_t stga_num_windows(int T, int Hg, int Wg, const int* w) {
  return ceil_div(T, w[0]) * ceil_div(Hg, w[1]) * ceil_div(Wg, w[2]);
}

// Encodes a 2-D bf16 tensor map (inner dim contiguous) with a 64 x box_rows
// box and 128-byte swizzle.  Returns false if the driver entry point is
// unavailable or the encoding fails.
bool make_tmap_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t row_stride_bytes,
                  uint32_t box_rows);
// Encodes a 3-D bf16 tensor map over [N tokens, H heads, d_h] (d_h innermost)
// with a box of 64 columns x 1 head x 128 tokens and 128-byte swizzle: one
// box is a 128-row operand tile of one head, read in place.
bool make_tmap_tokens(CUtensorMap* map, const void* base, uint64_t d_h, uint64_t H, uint64_t N);
// Encodes a 5-D bf16 tensor map over the (d_h, H, Wg, Hg, T) view of a
// [T*Hg*Wg, H, d_h] tensor with a box of 64 columns x 1 head x window[2] x
// window[1] x window[0] and 128-byte swizzle: one box is one STGA window of
// one head in the window's own (frame, row, column) order, with zeros where
// it leaves the grid.
bool make_tmap_box5(CUtensorMap* map, const void* base, uint64_t d_h, uint64_t H, uint64_t Wg, uint64_t Hg,
                    uint64_t T, const int* window);

}  // namespace moga
