/*
 * moga.h - C ABI of a single-GPU Mixture-of-Groups Attention (MoGA) layer for
 * NVIDIA B200 (sm_100a).
 *
 * Method: "MoGA: Mixture-of-Groups Attention for End-to-End Long Video
 * Generation" (arXiv 2510.18692), as summarised on the paper-graph-ui page of
 * that title, section 3.4 "Detailed, Sentence-Based Technical Breakdown":
 *   Eq. 1  SA(q, K, V) = softmax(q K^T / sqrt(d)) V              (Vanilla Self-Attention)
 *   Eq. 2  r = x W_r (+ b)                                       (MoGA Router)
 *   Eq. 3  p(i|x) = softmax(r)_i                                 (MoGA Router)
 *   Eq. 4  g(x) = argmax_i p(i|x)                                (MoGA Router)
 *   Eq. 5  MoGA(x) = p(g(x)|x) * SA(q, K_g(x), V_g(x))           (Grouped Attention)
 *   Algorithm 1: route; permute Q/K/V into per-group segments (cu_seqlen,
 *   max_seqlen, permute index); attention per segment; un-permute
 *                                                    (MoGA Pseudocode and Kernel Integration)
 *   STGA: attention inside fixed spatio-temporal windows; the block output is
 *   the mean of the MoGA and STGA outputs   (Spatial-Temporal Group Attention)
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensor pointers are DEVICE pointers, owned by the caller, 16-byte
 *   aligned and dense (row-major, no padding).  The library allocates no
 *   device memory: calls that need scratch take a caller-allocated workspace
 *   whose size comes from the matching *_workspace_size query.
 * - q, k, v and out are bf16 in [N, H, d_h] layout (token-major, then head,
 *   then channel).  d_h must be 64 or 128.
 * - x is [N, d] (fp32 or bf16), W_r is [M, d] in the same dtype (row i is
 *   group i's prototype, i.e. the nn.Linear weight layout; the d x M matrix of
 *   Eq. 2 is its transpose), b_r is an optional fp32 [M] bias.
 * - Softmax scale: 1/sqrt(d_h) per head.  Argmax ties go to the lowest group.
 * - perm[j] is the ORIGINAL index of the token at sorted position j; tokens
 *   are sorted by group, then by original index (stable), so perm is unique.
 *   offsets ("cu_seqlen") is int32 [M+1], offsets[0] = 0, offsets[M] = N.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  All work
 *   is enqueued asynchronously on it; a return of MOGA_OK means the work was
 *   validated and launched.  Errors found on the device (a bounded wait that
 *   timed out) are recorded in the workspace status word and reported by
 *   moga_sync_status().
 * - Arguments are validated before any device work is enqueued; an invalid
 *   argument returns MOGA_ERR_INVALID_ARG (or MOGA_ERR_UNSUPPORTED /
 *   MOGA_ERR_WORKSPACE) and touches nothing.
 * - N = 0 (no tokens) is legal wherever N is an argument: per-token buffers
 *   (x, q, k, v, out, group_id, gate, perm, and the gradient and branch
 *   outputs of the training calls) may then be NULL, offsets is set to zeros
 *   and nothing else is written.
 * - The library keeps no state between calls apart from cached kernel
 *   attributes, so distinct workspaces may be used from distinct threads.
 */
#ifndef MOGA_H_
#define MOGA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOGA_OK = 0,
  MOGA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or shape */
  MOGA_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d_h not 64/128) */
  MOGA_ERR_WORKSPACE = 3,     /* ws_bytes smaller than the size query returned */
  MOGA_ERR_CUDA = 4,          /* a CUDA runtime call or kernel launch failed */
  MOGA_ERR_TIMEOUT = 5,       /* a device-side bounded wait gave up */
  MOGA_ERR_DEVICE_CHECK = 6   /* a device-side range check fired */
} moga_status;

typedef enum { MOGA_F32 = 0, MOGA_BF16 = 1 } moga_dtype;

/* Human-readable name of a status code (static string, never NULL). */
const char* moga_status_string(int status);

/* ABI version: (major << 16) | minor. */
int moga_version(void);

/* ---------------------------------------------------------------- routing
 * moga_route: Eqs. 2-4 plus the index half of Algorithm 1, step 2.
 *   logits r = x W_r^T + b (fp32 accumulation), p = softmax(r),
 *   group_id[i] = argmax r (lowest index on ties), gate[i] = p(group_id[i]|x_i),
 *   offsets = exclusive prefix sum of the group sizes, max_seqlen = largest
 *   group, perm = stable sort of token indices by group.
 * In:  x [N, d] (dtype dt), W_r [M, d] (dtype dt), b_r [M] fp32 or NULL.
 * Out: group_id int32 [N], gate fp32 [N], perm int32 [N], offsets int32 [M+1],
 *      max_seqlen int32 [1] (device).
 * Limits: 0 <= N < 2^31, 1 <= M <= 1024, d >= 8 and d % 8 == 0 (bf16) or
 *         d % 4 == 0 (fp32).  N == 0 writes offsets = 0 and max_seqlen = 0.
 * Workspace: moga_route_workspace_size(N, M) bytes.
 */
size_t moga_route_workspace_size(int64_t N, int M);
moga_status moga_route(const void* x, const void* W_r, const float* b_r, moga_dtype dt, int64_t N, int d,
                       int M, int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets,
                       int32_t* max_seqlen, void* ws, size_t ws_bytes, void* stream);

/* moga_sort: the index half of Algorithm 1 step 2 for caller-given group ids
 * ("MoGA Pseudocode and Kernel Integration"): from group_id int32 [N] in
 * [0, M) it writes perm int32 [N] (stable: tokens by group, then by index),
 * offsets int32 [M+1] and max_seqlen int32 [1], exactly as moga_route does for
 * its own ids.  Ids outside [0, M) are skipped on the device (offsets[M] then
 * counts only valid tokens) and moga_sync_status() reports
 * MOGA_ERR_DEVICE_CHECK.  Used when routing happened elsewhere (e.g. on other
 * ranks of a sequence-parallel group).
 * Limits: 1 <= M <= 1024 (the same group limit as moga_route) and
 * 0 <= N < 2^31; anything else returns MOGA_ERR_INVALID_ARG before any launch.
 * Workspace: moga_sort_workspace_size(N, M) bytes. */
size_t moga_sort_workspace_size(int64_t N, int M);
moga_status moga_sort(const int32_t* group_id, int64_t N, int M, int32_t* perm, int32_t* offsets,
                      int32_t* max_seqlen, void* ws, size_t ws_bytes, void* stream);

/* moga_route_ex: moga_route plus the group-balancing statistics of the pages'
 * "Group Balancing Loss" section (Eq. 6), in the reading
 *   F_i = fraction of tokens routed to group i   (= (offsets[i+1]-offsets[i])/N)
 *   P_i = (1/N) * sum over all tokens x of p(i|x)
 *   balance = M * sum_i F_i P_i               (1 when balanced and confident)
 * prob_mean (fp32 [M], device) receives P, balance (fp32 [1], device) the
 * metric; either may be NULL (both NULL = plain moga_route).  The sums are
 * taken in a fixed order, so the results are deterministic.
 * Workspace: moga_route_ex_workspace_size(N, M) bytes. */
size_t moga_route_ex_workspace_size(int64_t N, int M);
moga_status moga_route_ex(const void* x, const void* W_r, const float* b_r, moga_dtype dt, int64_t N, int d, int M,
                          int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets, int32_t* max_seqlen,
                          float* prob_mean, float* balance, void* ws, size_t ws_bytes, void* stream);

/* moga_route_noalloc: the same routing as moga_route, for callers that cannot
 * allocate device memory themselves (for example code running inside a
 * framework whose allocator owns the GPU, or a pre-recorded launch sequence
 * that must not call cudaMalloc).  It takes no workspace: its scratch (the
 * per-tile group histograms and bases, about 2 MiB) is a fixed device array
 * inside the library that every GPU loading the library keeps until the
 * process exits.  The method pages have no counterpart to this call; it only
 * changes where the scratch lives.
 * - Outputs, limits and results are those of moga_route, plus one more limit:
 *   ceil(N / 128) * M <= 262144 (e.g. N = 580,320 with M = 32, or N = 187,200
 *   with M = 64); larger sizes return MOGA_ERR_WORKSPACE and touch nothing.
 * - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture on the device.  The address is kept per device
 *   and context, so a call after a device reset looks it up again.
 * - Every call shares the one array and it keeps the last call's contents;
 *   the call clears what must start at zero.  Calls that overlap on the GPU
 *   (different streams, or different host threads, on one device) race on
 *   the array: order them on one stream.
 * - Device-side conditions (a bounded wait that ran out, ids out of range)
 *   go to a status word at the head of the array; read them with
 *   moga_route_noalloc_status. */
moga_status moga_route_noalloc(const void* x, const void* W_r, const float* b_r, moga_dtype dt, int64_t N, int d,
                               int M, int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets,
                               int32_t* max_seqlen, void* stream);

/* moga_route_noalloc_status: synchronises the stream, then reads and clears
 * the device status word of moga_route_noalloc's scratch on the current
 * device (MOGA_OK, MOGA_ERR_TIMEOUT or MOGA_ERR_DEVICE_CHECK, as
 * moga_sync_status does for a workspace).  Allocates nothing. */
moga_status moga_route_noalloc_status(void* stream);

/* ---------------------------------------------------------------- grouped attention
 * moga_group_attn: Algorithm 1 steps 2 (gather Q/K/V into group order), 3
 * (attention inside each group segment) and 4 (un-permute), with the gate of
 * Eq. 5 fused into the store:   out[perm[j], h, :] = out_scale * gate[perm[j]] *
 *              SA(q[perm[j],h], K_seg(j),h, V_seg(j),h)
 * where seg(j) is the segment of offsets that contains j.  gate may be NULL
 * (gate = 1).  Tokens of empty groups do not exist, so every token's row of
 * `out` is written exactly once.
 * In:  q, k, v bf16 [N, H, d_h]; perm int32 [N]; offsets int32 [M+1]
 *      (non-decreasing, offsets[0] = 0, offsets[M] = N); gate fp32 [N] or
 *      NULL.  The device checks offsets and every perm entry it uses: a
 *      violation skips the affected work and is reported by
 *      moga_sync_status() as MOGA_ERR_DEVICE_CHECK.
 * Out: out bf16 [N, H, d_h].
 * Limits: d_h in {64, 128}; 1 <= H; N * H < 2^31; 1 <= M <= 1024.
 * Workspace: moga_group_attn_workspace_size(N, H, d_h, M) bytes.
 */
size_t moga_group_attn_workspace_size(int64_t N, int H, int d_h, int M);
moga_status moga_group_attn(const void* q, const void* k, const void* v, const int32_t* perm,
                            const int32_t* offsets, const float* gate, int64_t N, int H, int d_h, int M,
                            float out_scale, void* out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- STGA windows
 * stga_window_attn: full attention inside non-overlapping windows of
 * window[0] x window[1] x window[2] (frames x rows x columns) tokens over the
 * T x Hg x Wg latent grid, windows anchored at the grid origin and clipped at
 * the edges; token index = (t * Hg + h) * Wg + w.
 *   accumulate == 0: out = STGA(q, k, v)
 *   accumulate == 1: out = out + 0.5 * STGA(q, k, v)   (second half of the
 *                    two-branch mean; the caller wrote 0.5 * MoGA before)
 * In:  q, k, v bf16 [N, H, d_h], N = T * Hg * Wg.   Out: out bf16 [N, H, d_h].
 * Limits: as moga_group_attn; every window extent >= 1.
 * Workspace: stga_window_attn_workspace_size(...) bytes.
 */
size_t stga_window_attn_workspace_size(int T, int Hg, int Wg, const int* window, int H, int d_h);
moga_status stga_window_attn(const void* q, const void* k, const void* v, int T, int Hg, int Wg,
                             const int* window, int H, int d_h, int accumulate, void* out, void* ws,
                             size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- shot-aware STGA
 * stga_shot_attn: the STGA branch with shots ("Spatial-Temporal Group
 * Attention (STGA)" section: frames of different shots are in distinct
 * temporal groups; keys and values, not queries, are augmented with latent
 * frames of the adjacent shots).  Reading taken:
 *   - shot_start (DEVICE int32 [nshots + 1]): 0 = s_0 < s_1 < ... < s_nshots
 *     = T; shot j holds latent frames [s_j, s_{j+1}).  Checked on the device:
 *     a violation skips all work and moga_sync_status() reports
 *     MOGA_ERR_DEVICE_CHECK.
 *   - window (host int[3]) = (wt, wh, ww): temporal windows of wt frames tile
 *     each shot from its first frame and are clipped at its last; wt = 0 makes
 *     one temporal window per shot (the pages' Wan setting is (0, Hg/2, Wg/2),
 *     a 2x2 spatial partition).  Spatial tiles as in stga_window_attn.
 *   - the keys/values of a shot's first temporal window add the previous
 *     shot's last aug_prev frames, those of its last temporal window the next
 *     shot's first aug_next frames (each clipped to that shot), in the same
 *     spatial tile; the pages' choice is aug_prev = aug_next = 2.
 * accumulate = 0: out = out_scale * SA; accumulate = 1: out += out_scale * SA
 * (the block's mean of branches).  q, k, v, out: bf16 [T*Hg*Wg, H, d_h].
 * Workspace: stga_shot_attn_workspace_size(...) bytes (an upper bound that
 * holds for every split of T frames into nshots shots).
 */
size_t stga_shot_attn_workspace_size(int T, int Hg, int Wg, const int* window, int nshots, int aug_prev,
                                     int aug_next, int H, int d_h);
moga_status stga_shot_attn(const void* q, const void* k, const void* v, int T, int Hg, int Wg, const int* window,
                           const int32_t* shot_start, int nshots, int aug_prev, int aug_next, int H, int d_h,
                           float out_scale, int accumulate, void* out, void* ws, size_t ws_bytes, void* stream);

/* moga_layer_shots: the visual block of the pages' Wan setting, one call:
 * moga_route, grouped attention, shot-aware STGA (stga_shot_attn with the
 * given window, shots and augmentation) and, when per_frame = 1, the
 * per-frame branch; out = arithmetic mean of the branches (2 or 3 of them).
 * Arguments and outputs as moga_layer_ex and stga_shot_attn (shot_start is
 * device int32 [nshots + 1]; T * Hg * Wg must equal N).
 * Workspace: moga_layer_shots_workspace_size(...) bytes. */
size_t moga_layer_shots_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg, const int* window,
                                       int nshots, int aug_prev, int aug_next, int per_frame);
moga_status moga_layer_shots(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                             const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                             int Wg, const int* window, const int32_t* shot_start, int nshots, int aug_prev,
                             int aug_next, int per_frame, void* out, int32_t* group_id, float* gate, int32_t* perm,
                             int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- full layer
 * moga_layer: one visual attention block = moga_route, then moga_group_attn,
 * then (when window != NULL) stga_window_attn, combined as
 *   out = 0.5 * (MoGA(x) + STGA(x))   (window != NULL)
 *   out = MoGA(x)                     (window == NULL; T, Hg, Wg ignored)
 * All outputs (out, group_id, gate, perm, offsets) are caller-owned device
 * buffers with the shapes given above.
 * Workspace: moga_layer_workspace_size(...) bytes.
 */
size_t moga_layer_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg, const int* window);
moga_status moga_layer(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                       const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                       int Wg, const int* window, void* out, int32_t* group_id, float* gate, int32_t* perm,
                       int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- training
 * moga_layer_train: the forward of moga_layer that keeps what the backward
 * pass needs.  Outputs as moga_layer plus
 *   o_moga   bf16 [N, H, d_h]  MoGA branch alone, gate * SA (Eq. 5)
 *   o_stga   bf16 [N, H, d_h]  STGA branch alone (window != NULL; else unused)
 *   lse_moga fp32 [H, N]       natural-log log-sum-exp of each query's scaled
 *                              scores q.k/sqrt(d_h) within its group, at the
 *                              token's sorted position (perm order)
 *   lse_stga fp32 [H, N]       the same within its STGA window, in window
 *                              order (windows as in stga_window_attn, tokens
 *                              of a window in index order)
 *   out = 0.5 * (o_moga + o_stga), or o_moga when window == NULL (out may then
 *   be o_moga itself; with a window the three outputs must be distinct).
 * Workspace: moga_layer_train_workspace_size(...) bytes. */
size_t moga_layer_train_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg, const int* window);
moga_status moga_layer_train(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                             const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                             int Wg, const int* window, void* out, void* o_moga, void* o_stga, float* lse_moga,
                             float* lse_stga, int32_t* group_id, float* gate, int32_t* perm, int32_t* offsets,
                             void* ws, size_t ws_bytes, void* stream);

/* moga_layer_backward: gradients of a scalar loss L through the block, given
 * dout = dL/dout (bf16 [N, H, d_h]) and what moga_layer_train returned
 * ("MoGA Router" and "Grouped Attention" sections: the argmax assignment is
 * not differentiable; the router learns through the gate p(g(x)|x) of Eq. 5,
 * q, k, v through the attention of each branch with the assignment held
 * fixed).  With w = 1/2 (window != NULL) or 1:
 *   dq, dk, dv  bf16 [N, H, d_h]: w * gate * dout through MoGA's attention
 *               plus w * dout through STGA's (overwritten, not accumulated);
 *   dgate_i   = w * sum_{h,c} dout * o_moga / gate_i;
 *   dr_ij     = dgate_i * p_ig * ([j == g_i] - p_ij) for the router's
 *               softmax p = softmax(x W_r^T + b), recomputed by the
 *               forward's router kernel (the same logits bit for bit);
 *   dx        = dr W_r   (x's dtype, [N, d]: the router's share of dL/dx;
 *               q, k, v are inputs of the block, so the projections that
 *               produce them are the caller's);
 *   dW_r      = dr^T x   (fp32 [M, d], overwritten);
 *   db_r      = sum_i dr_i (fp32 [M], overwritten; may be NULL).
 * The inputs (x, W_r, b_r, q, k, v, group_id, gate, perm, offsets, o_moga,
 * o_stga, lse_*) must be those of the forward call.  dW_r and db_r are
 * summed in a fixed order (deterministic); bf16 outputs are rounded once per
 * branch (the STGA share is added to the MoGA share in bf16).
 * Workspace: moga_layer_backward_workspace_size(N, d, H, d_h, M) bytes
 * (head-major copies of q, k, v and dO, plus per-token scratch). */
size_t moga_layer_backward_workspace_size(int64_t N, int d, int H, int d_h, int M);
moga_status moga_layer_backward(const void* dout, const void* x, const void* W_r, const float* b_r, moga_dtype x_dt,
                                const void* q, const void* k, const void* v, int64_t N, int d, int H, int d_h, int M,
                                int T, int Hg, int Wg, const int* window, const void* o_moga, const void* o_stga,
                                const float* lse_moga, const float* lse_stga, const int32_t* group_id,
                                const float* gate, const int32_t* perm, const int32_t* offsets, void* dx,
                                float* dW_r, float* db_r, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                void* stream);

/* moga_layer_train_ex / moga_layer_backward_ex: the same pair with the
 * per-frame branch of the "Spatial-Temporal Group Attention (STGA)" section
 * as a third branch (per_frame = 1: attention among all Hg*Wg tokens of each
 * latent frame; T, Hg, Wg are then required even when window == NULL).
 * out is the plain mean of the branches that are on, and each branch's share
 * of dout in the backward is dout divided by their number.  o_frame (bf16
 * [N, H, d_h]) and lse_frame (fp32 [H, N], token order) are the per-frame
 * branch's output and log-sum-exp, unused when per_frame = 0.  Everything
 * else as moga_layer_train / moga_layer_backward (which are these calls with
 * per_frame = 0 and balance_alpha = 0).
 * balance_alpha (finite): adds the group balancing loss of the "Group
 * Balancing Loss" section, alpha * M * sum_i F_i P_i with F_i the share of
 * tokens routed to group i (from offsets; an argmax count, so it carries no
 * gradient) and P_i the mean over tokens of p(i|x), to the loss whose router
 * gradient is returned: dr_ij += alpha * M / N * p_ij * (F_j - sum_k F_k p_ik).
 * 0 leaves it out.
 * Workspace: moga_layer_train_ex_workspace_size(...) / moga_layer_backward_workspace_size(...). */
size_t moga_layer_train_ex_workspace_size(int64_t N, int H, int d_h, int M, int T, int Hg, int Wg,
                                          const int* window, int per_frame);
moga_status moga_layer_train_ex(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                                const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                                int Wg, const int* window, int per_frame, void* out, void* o_moga, void* o_stga,
                                void* o_frame, float* lse_moga, float* lse_stga, float* lse_frame, int32_t* group_id,
                                float* gate, int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes,
                                void* stream);
moga_status moga_layer_backward_ex(const void* dout, const void* x, const void* W_r, const float* b_r,
                                   moga_dtype x_dt, const void* q, const void* k, const void* v, int64_t N, int d,
                                   int H, int d_h, int M, int T, int Hg, int Wg, const int* window, int per_frame,
                                   float balance_alpha, const void* o_moga, const void* o_stga, const void* o_frame,
                                   const float* lse_moga,
                                   const float* lse_stga, const float* lse_frame, const int32_t* group_id,
                                   const float* gate, const int32_t* perm, const int32_t* offsets, void* dx,
                                   float* dW_r, float* db_r, void* dq, void* dk, void* dv, void* ws, size_t ws_bytes,
                                   void* stream);

/* moga_layer_ex: the visual block with a choice of branches, as in the pages'
 * "Spatial-Temporal Group Attention (STGA)" section (each token's output is
 * the mean of its MoGA group, its STGA window and its per-frame group):
 *   branches bit 0: the STGA window branch (window required),
 *   branches bit 1: the per-frame branch, attention among all tokens of each
 *                   latent frame (window 1 x Hg x Wg),
 *   out = arithmetic mean of MoGA(x) and the branches that are on.
 * branches = 1 is moga_layer with a window, branches = 0 is MoGA alone.
 * Other arguments, outputs and limits as moga_layer; T, Hg, Wg are required
 * whenever branches != 0.
 * Workspace: moga_layer_ex_workspace_size(N, H, d_h, M, branches) bytes. */
size_t moga_layer_ex_workspace_size(int64_t N, int H, int d_h, int M, int branches);
moga_status moga_layer_ex(const void* x, const void* W_r, const float* b_r, moga_dtype x_dt, const void* q,
                          const void* k, const void* v, int64_t N, int d, int H, int d_h, int M, int T, int Hg,
                          int Wg, const int* window, int branches, void* out, int32_t* group_id, float* gate,
                          int32_t* perm, int32_t* offsets, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------- host pipeline
 * A pipeline runs the visual block of moga_layer_ex (same arithmetic, same
 * branches) on inputs that live in HOST memory and returns the output to host
 * memory, step after step, with the copies of one step overlapping the
 * compute of its neighbours: step i+1's inputs travel host -> device while
 * step i computes and step i-1's output travels back.  It owns two device
 * slots of inputs and outputs, one workspace and three streams (copy in,
 * compute, copy out), all on the device that is current at creation.
 * Host buffers should be page-locked (cudaHostAlloc / cudaHostRegister): the
 * copies are then asynchronous DMA; pageable memory still works but the copies
 * stop overlapping.  The pipeline is not thread-safe: one host thread at a time.
 *
 * moga_pipe_create: shapes and branches as moga_layer_ex (window required when
 * branches & 1; T, Hg, Wg required when branches != 0).  Allocates about
 * 2 x (inputs + outputs) + the layer workspace of device memory.
 * On success *pipe receives the handle.  Invalid shapes return
 * MOGA_ERR_INVALID_ARG / MOGA_ERR_UNSUPPORTED before any CUDA call.
 */
typedef struct moga_pipe moga_pipe;
moga_status moga_pipe_create(int64_t N, int d, int H, int d_h, int M, moga_dtype x_dt, int T, int Hg, int Wg,
                             const int* window, int branches, moga_pipe** pipe);

/* moga_pipe_submit: enqueues one step and returns without waiting.
 * In (host): x [N, d] (x_dt), W_r [M, d] (x_dt), b_r fp32 [M] or NULL,
 *            q, k, v bf16 [N, H, d_h].
 * Out (host): out bf16 [N, H, d_h]; group_id int32 [N] and gate fp32 [N]
 *            optional (NULL = not returned).
 * Every host buffer must stay valid, and the inputs unchanged, until
 * moga_pipe_sync() returns; the outputs hold the step's result from then on.
 * Returns MOGA_ERR_INVALID_ARG for a NULL required pointer or a NULL pipe, and
 * MOGA_ERR_CUDA if enqueueing failed. */
moga_status moga_pipe_submit(moga_pipe* pipe, const void* x, const void* W_r, const float* b_r, const void* q,
                             const void* k, const void* v, void* out, int32_t* group_id, float* gate);

/* moga_pipe_sync: waits for every submitted step, then reads and clears the
 * device status word; returns MOGA_OK, MOGA_ERR_TIMEOUT, MOGA_ERR_DEVICE_CHECK
 * or MOGA_ERR_CUDA (the first error of any step since the last sync). */
moga_status moga_pipe_sync(moga_pipe* pipe);

/* moga_pipe_destroy: waits for outstanding steps and frees everything.
 * NULL is a no-op. */
moga_status moga_pipe_destroy(moga_pipe* pipe);

/* ---------------------------------------------------------------- device status
 * moga_sync_status: synchronises `stream`, reads the device status word kept
 * at the start of a workspace `ws` used by the calls above, clears it, and
 * returns MOGA_OK, MOGA_ERR_TIMEOUT or MOGA_ERR_DEVICE_CHECK (or MOGA_ERR_CUDA
 * if the synchronisation itself failed).  Workspaces must be zero-filled once
 * before first use so that the status word starts clear.
 */
moga_status moga_sync_status(void* ws, void* stream);

/* moga_set_wait_limit_ns: upper bound, in nanoseconds, on any single
 * device-side wait of the kernels launched after this call (default 4e9).
 * Process-wide.  Returns the previous value. */
uint64_t moga_set_wait_limit_ns(uint64_t ns);

/* ---------------------------------------------------------------- instrumentation
 * moga_kernel_launches: process-wide count of kernels this library has
 * launched so far (memsets excluded).
 *
 * moga_set_timing_events: when begin/end are non-NULL cudaEvent_t handles,
 * every later call records `begin` on its stream right before the launches of
 * `stage` and `end` right after them (so the event pair brackets exactly that
 * stage's kernels on the stream they run on).  NULL/NULL detaches.  Process-
 * wide and not synchronised with concurrent calls: meant for benchmarks.
 * Returns MOGA_ERR_INVALID_ARG for an unknown stage or a half-NULL pair. */
typedef enum {
  MOGA_STAGE_ROUTER = 0,      /* router kernel (logits, gate, argmax, tile histogram) */
  MOGA_STAGE_SORT = 1,        /* scan + stable scatter -> offsets, perm */
  MOGA_STAGE_GATHER = 2,      /* segment table + gather of Q/K/V into group order */
  MOGA_STAGE_GROUP_ATTN = 3,  /* grouped attention kernel (incl. gate + un-permute) */
  MOGA_STAGE_STGA_PREP = 4,   /* window-order permutation (+ gather for windows over 256 tokens) */
  MOGA_STAGE_STGA_ATTN = 5    /* STGA window attention kernel (incl. the mean) */
} moga_stage;
uint64_t moga_kernel_launches(void);
moga_status moga_set_timing_events(int stage, void* begin, void* end);

/* moga_debug_inject: failure-detection test hook, process-wide.
 *   0: off (default).
 *   1: in later attention calls (grouped, STGA, shot-aware, and the layers
 *      built on them), the attention kernel's loader withholds each CTA's
 *      first K tile, so the MMA warp's bounded wait runs out: the kernel
 *      drains, frees its tensor memory and exits, and moga_sync_status()
 *      reports MOGA_ERR_TIMEOUT.  Nothing faults
 *      or hangs; the CUDA context stays usable.  Pair with a short
 *      moga_set_wait_limit_ns().
 * Returns MOGA_ERR_INVALID_ARG for other modes. */
moga_status moga_debug_inject(int mode);

#ifdef __cplusplus
}
#endif
#endif /* MOGA_H_ */
