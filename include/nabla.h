/*
 * nabla.h -- C ABI of libnabla.so: NABLA block-sparse 3D self-attention for
 * video diffusion transformers, on NVIDIA B200 (sm_100a).
 *
 * The method is the one described in "NABLA: Neighborhood Adaptive Block-Level
 * Attention" (gist.science technical summary, section 手法: NABLA):
 *   1. fractal flattening of the T x H x W token grid (P x P patches made
 *      contiguous, time order kept)                      -> nabla_flatten
 *   2. mean-pooling Q and K into blocks of P*P tokens, the full attention map
 *      over the pooled blocks, a per-row CDF cut at mass p, OR with a static
 *      Sliding-Tile window (M = M_nabla OR M_STA)           -> nabla_build_mask
 *   3. attention computed exactly on the kept blocks     -> nabla_attn_fwd
 *   4. its gradients for training                        -> nabla_attn_bwd
 *
 * Conventions shared by every call
 *   - All tensors live in device memory that the CALLER allocated; the library
 *     allocates nothing and keeps no state between calls.  Scratch memory is
 *     the caller's workspace, sized by nabla_workspace_size().  The one
 *     exception is nabla_build_mask_static, whose scratch is an array compiled
 *     into the library (held per GPU until exit) and which caches that array's
 *     device address per device.
 *   - Every call only enqueues work on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream) and returns without synchronising the host.
 *     Errors found on the host (shape, alignment, parameters, workspace size,
 *     launch failure) are returned immediately and nothing is enqueued.
 *     A device-side failure (a bounded wait that expired) is written to the
 *     status word at the start of the workspace; read it with nabla_status().
 *   - Q, K, V, O, dO, dQ, dK, dV are bf16 (raw 16-bit patterns, nabla_bf16),
 *     contiguous [B, heads, N, D] with N = T*H*W tokens in FLATTENED order.
 *   - Pointers to tensors must be 16-byte aligned (NABLA_ERR_ALIGN).
 *   - Supported: P = 8 (blocks of 64 tokens), D in {64, 128}, H and W
 *     multiples of P, 1 <= number of blocks nb = T*(H/P)*(W/P) <= 2048.
 *
 * Return value of every int function: NABLA_OK (0) or a negative status.
 */
#ifndef NABLA_H
#define NABLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t nabla_bf16;               /* raw bf16 bit pattern */
typedef struct CUstream_st *nabla_stream_t; /* == cudaStream_t */

#define NABLA_OK 0
#define NABLA_ERR_SHAPE (-1)     /* grid not divisible by P, unsupported D, P or nb */
#define NABLA_ERR_ALIGN (-2)     /* pointer not 16-byte aligned, inner_bytes % 16 != 0 */
#define NABLA_ERR_PARAM (-3)     /* p not in [0,1], STA window even or < 1, scale <= 0 */
#define NABLA_ERR_WORKSPACE (-4) /* workspace missing or smaller than required */
#define NABLA_ERR_CUDA (-5)      /* a CUDA call or kernel launch failed */
#define NABLA_ERR_TIMEOUT (-6)   /* a device-side bounded wait expired */
#define NABLA_ERR_NULL (-7)      /* a required pointer is NULL */

/* nabla_params.flags */
#define NABLA_NO_STA 1u    /* no STA term: M = adaptive OR diagonal            */
#define NABLA_FULL_STA 2u  /* STA window covers every block: dense attention   */
#define NABLA_EMIT_COLS 4u /* also write the column lists needed by the backward */
/* Also write the pooled block scores s_ij (float32, [B*heads, nb, nb]) into
 * mask->scores, exactly as the cut used them, so that a caller can re-run the
 * cut on them (a check of the score phase).  Written only when the mask
 * depends on the scores (0 < p < 1 and not NABLA_FULL_STA). */
#define NABLA_DEBUG_SCORES 8u
/* Test aid, not for production: makes the tensor-core attention forward and
 * backward, and the persistent front end of nabla_build_mask_grid, give up a
 * device-side wait at once (or after 1 ms), so that the timeout path (status
 * word = NABLA_ERR_TIMEOUT, clean unwind, context still usable) can be
 * exercised without faulting or hanging the GPU.  Outputs are not meaningful
 * after it. */
#define NABLA_DEBUG_TIMEOUT 0x100u

/* Problem shape.  P must be 8. */
typedef struct {
    int B, heads, T, H, W, D, P;
} nabla_shape;

/* Mask / attention parameters.
 *   p      CDF mass threshold in [0, 1] ("thr" on the page).  Per row, the
 *          kept adaptive set is the shortest run of blocks, taken in
 *          descending pooled score (equal scores: lower index first), whose
 *          softmax mass reaches p; p = 1 keeps every block, p = 0 none.
 *   sta_t, sta_h, sta_w  odd STA window, in blocks (frames, patch rows,
 *          patch columns), centred, truncated at the grid border.
 *   scale  softmax scale of both the pooled map and the attention
 *          (usually 1/sqrt(D)).
 *   flags  NABLA_NO_STA | NABLA_FULL_STA | NABLA_EMIT_COLS |
 *          NABLA_DEBUG_SCORES (and the test aid NABLA_DEBUG_TIMEOUT). */
typedef struct {
    float p;
    int sta_t, sta_h, sta_w;
    float scale;
    unsigned flags;
} nabla_params;

/* Block mask M, caller-allocated (sizes from nabla_mask_bytes), device memory.
 *   bits    [B*heads, nb, ceil(nb/32)] uint32: bit (j % 32) of word j / 32 of
 *           row i is set when block j is kept for query block i.
 *   row_idx [B*heads, nb, nb] uint16: kept j of row i, ascending; only the
 *           first row_cnt entries of each row are written.
 *   row_cnt [B*heads, nb] int32.
 *   col_idx, col_cnt: the transpose (query blocks i keeping key block j,
 *           ascending i); written only with NABLA_EMIT_COLS, required by
 *           nabla_attn_bwd.  May be NULL otherwise.
 *   scores  [B*heads, nb, nb] float32 pooled scores; written only with
 *           NABLA_DEBUG_SCORES (then required), may be NULL otherwise. */
typedef struct {
    uint32_t *bits;
    uint16_t *row_idx;
    int32_t *row_cnt;
    uint16_t *col_idx;
    int32_t *col_cnt;
    float *scores;
} nabla_mask;

/* Which part of the mask nabla_mask_bytes() sizes. */
#define NABLA_MASK_BITS 0
#define NABLA_MASK_ROW_IDX 1
#define NABLA_MASK_ROW_CNT 2
#define NABLA_MASK_COL_IDX 3
#define NABLA_MASK_COL_CNT 4
#define NABLA_MASK_SCORES 5

/* Which call nabla_workspace_size() sizes. */
#define NABLA_OP_BUILD_MASK 0
#define NABLA_OP_ATTN_FWD 1
#define NABLA_OP_ATTN_BWD 2

/* Fractal flattening (section 手法: NABLA, "トークン再順序付け (Fractal
 * Flattening)").  `in` and `out` are [outer, T, H, W, inner_bytes] in grid
 * order and [outer, N, inner_bytes] in flattened order, where token (t, y, x)
 * goes to
 *   n = ((t*(H/P) + y/P)*(W/P) + x/P)*P*P + (y%P)*P + x%P
 * (one level of P x P patches, patch grid and patch interior row-major).
 * inverse = 0 maps grid -> flattened, inverse = 1 flattened -> grid.
 * Any P >= 1 dividing H and W; inner_bytes % 16 == 0; in and out must not
 * overlap (NABLA_ERR_PARAM; no in-place).  Works for [B, T, H, W, C]
 * activations and [B*h, T, H, W, D] heads alike. */
int nabla_flatten(const void *in, void *out, int64_t outer, int T, int H, int W, int P,
                  int64_t inner_bytes, int inverse, nabla_stream_t stream);

/* Bytes of workspace `op` needs for `shape` (0 for an invalid shape).
 * Every workspace starts with a 256-byte status region. */
size_t nabla_workspace_size(const nabla_shape *shape, int op);

/* Bytes of mask part `part` (NABLA_MASK_*) for `shape` (0 if invalid). */
size_t nabla_mask_bytes(const nabla_shape *shape, int part);

/* Build M from flattened q, k (section 手法: NABLA, "適応型マスク構築" and
 * "STA とのハイブリッド統合").  Per (batch, head) and query block i:
 *   qbar_i, kbar_j = means of the 64 tokens of block i / j, summed in float32
 *                    in ascending token order, times 1/64;
 *   s_ij           = float32 fused multiply-add chain over d ascending, times
 *                    scale;
 *   w_ij           = exp(s_ij - max_j s_ij) in float64, mass u_ij =
 *                    floor(w_ij * 2^40) as an exact integer;
 *   adaptive set   = shortest prefix of j ordered by (s_ij desc, j asc) whose
 *                    summed u reaches p * sum_j u_ij (float64 product);
 *   M_ij           = adaptive OR STA window OR (i == j).
 * Writes bits, row lists, (with NABLA_EMIT_COLS) column lists and (with
 * NABLA_DEBUG_SCORES) the scores s_ij.
 * When M does not depend on the scores -- p >= 1 or NABLA_FULL_STA (every
 * block), p <= 0 (STA window and diagonal; the diagonal alone with
 * NABLA_NO_STA) -- q and k are not read and no pooling or scores are computed
 * (the pure-STA configuration runs at list-emission cost); the arguments are
 * validated as usual.
 * Workspace: nabla_workspace_size(shape, NABLA_OP_BUILD_MASK) bytes, 256-byte
 * aligned. */
int nabla_build_mask(const nabla_shape *shape, const nabla_params *params,
                     const nabla_bf16 *q, const nabla_bf16 *k, const nabla_mask *mask,
                     void *workspace, size_t workspace_bytes, nabla_stream_t stream);

/* Flattening of Q and K fused with the mask build (sections 手法: NABLA,
 * "トークン再順序付け (Fractal Flattening)" and "適応型マスク構築"): the
 * same outputs as nabla_flatten(q_grid -> q), nabla_flatten(k_grid -> k)
 * followed by nabla_build_mask(q, k), with the pooling done in the flattening
 * pass instead of re-reading the flattened copies, and the flattening of one
 * head running beside the scores and cut of the previous one (one persistent
 * launch; its device-side waits are bounded and report NABLA_ERR_TIMEOUT
 * through nabla_status()).
 *   q_grid, k_grid  [B, heads, T, H, W, D] bf16 in grid order (inputs);
 *   q, k            [B, heads, N, D] bf16, written in flattened order (outputs;
 *                   the attention calls take them);
 *   mask, workspace as nabla_build_mask; the pooled means are bit-identical.
 * q and k must not overlap each other or either input (NABLA_ERR_PARAM).  All
 * four pointers 16-byte aligned.  Other checks as nabla_build_mask. */
int nabla_build_mask_grid(const nabla_shape *shape, const nabla_params *params,
                          const nabla_bf16 *q_grid, const nabla_bf16 *k_grid, nabla_bf16 *q,
                          nabla_bf16 *k, const nabla_mask *mask, void *workspace,
                          size_t workspace_bytes, nabla_stream_t stream);

/* Same computation and outputs as nabla_build_mask, without a workspace.
 * (No counterpart on the page: this is a calling convenience.)
 *
 * For callers that are handed only their input and output buffers and cannot
 * call cudaMalloc -- for example a plugin interface that passes no workspace,
 * or a process whose device memory is reserved up front by another allocator
 * -- so cannot provide the scratch nabla_build_mask needs for the pooled
 * means.  Here that scratch is a 32 MiB array compiled into the library: every
 * GPU that loads the library holds those 32 MiB until the process exits.
 *   - Limit: round_up_256(4 * B*heads * nb * D) + round_up_256(4 * B*heads * D *
 *     round_up_4(nb)) <= 32 MiB (e.g. 16 heads of a 1440-block, D = 128
 *     problem fit; 40 heads of 1200 blocks do not).
 *     Larger shapes return NABLA_ERR_WORKSPACE and enqueue nothing.
 *   - The first call on a device (the current device) looks up the array's
 *     device address with cudaGetSymbolAddress; make that first call before
 *     any stream capture on that device.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - All calls share the one array per device, which keeps the last call's
 *     contents.  Calls whose GPU work overlaps (other streams, other host
 *     threads) race on it; serialise them.  Nothing in the array needs to
 *     start at zero: each call writes every scratch byte it reads.
 *   - cudaDeviceReset invalidates the cached address: after resetting a
 *     device, do not call this entry point on it again in the same process.
 * Other arguments, checks and outputs: as nabla_build_mask. */
int nabla_build_mask_static(const nabla_shape *shape, const nabla_params *params,
                            const nabla_bf16 *q, const nabla_bf16 *k, const nabla_mask *mask,
                            nabla_stream_t stream);

/* DynamicRad-style masks in the same format ("DynamicRad: Content-Adaptive
 * Sparse Attention for Long Video Diffusion", section 2.A "Dual-Mode
 * Strategy"): a second pair of mask producers for the same attention calls.
 * Per (batch, head) and query block i = (t_i, ph_i, pw_i):
 *   NABLA_DR_STATIC_RATIO (content-free; q and k are not read, may be NULL):
 *     in frame t_j, with dt = |t_j - t_i|, keep the
 *       k(dt) = ceil(min(1, max(lambda, gamma^dt)) * Hp * Wp)
 *     patches nearest to (ph_i, pw_i): ascending (ph - ph_i)^2 + (pw - pw_i)^2,
 *     equal distances by ascending block index.  gamma^dt is a product of dt
 *     factors in float64 and k a float64 product rounded up.
 *   NABLA_DR_THRESHOLD (content-adaptive): with the pooled scores s_ij of
 *     nabla_build_mask (same float32 arithmetic), keep j where the float32
 *     difference max_j s_ij - s_ij <= tau: the blocks whose pre-softmax logit
 *     is within tau of the row's best (softmax weight >= e^-tau of the best).
 *   M_ij = selected OR STA window (unless NABLA_NO_STA) OR (i == j).
 * gamma in (0, 1], lambda in [0, 1], tau >= 0 (infinity keeps everything);
 * other fields and flags (NABLA_NO_STA, NABLA_EMIT_COLS, NABLA_DEBUG_SCORES in
 * the threshold mode) as nabla_params.  Workspace: as nabla_build_mask for
 * the threshold mode; the static mode needs only the status region
 * (nabla_workspace_size(shape, NABLA_OP_ATTN_FWD) bytes suffice). */
#define NABLA_DR_STATIC_RATIO 0
#define NABLA_DR_THRESHOLD 1
typedef struct {
    int mode;
    double gamma, lambda;
    float tau;
    int sta_t, sta_h, sta_w;
    float scale;
    unsigned flags;
} nabla_dr_params;

int nabla_build_mask_dr(const nabla_shape *shape, const nabla_dr_params *params,
                        const nabla_bf16 *q, const nabla_bf16 *k, const nabla_mask *mask,
                        void *workspace, size_t workspace_bytes, nabla_stream_t stream);

/* Block-sparse attention forward over M (bullet "拡張": attention is
 * computed for the kept blocks only).  For query token n of block i:
 *   o_n   = sum over tokens m of blocks j in row i of M of
 *           softmax_m(scale * q_n . k_m) v_m          (bf16 out, fp32 accumulate)
 *   lse_n = log sum_m exp(scale * q_n . k_m)          (float32 [B*heads, N])
 * Needs mask->bits, mask->row_idx and mask->row_cnt.  lse may be NULL when
 * no backward follows.  Workspace: nabla_workspace_size(shape,
 * NABLA_OP_ATTN_FWD).  Runs on the tcgen05 tensor cores; a device-side
 * wait that expires (it never should) is reported through nabla_status() and
 * leaves O and lse unwritten. */
int nabla_attn_fwd(const nabla_shape *shape, const nabla_params *params, const nabla_bf16 *q,
                   const nabla_bf16 *k, const nabla_bf16 *v, const nabla_mask *mask,
                   nabla_bf16 *o, float *lse, void *workspace, size_t workspace_bytes,
                   nabla_stream_t stream);

/* Gradients of nabla_attn_fwd (training through NABLA):
 *   D_n = dO_n . o_n,  P_nm = exp(scale q_n.k_m - lse_n),
 *   dV_m = sum_n P_nm dO_n,  dS_nm = P_nm (dO_n . v_m - D_n),
 *   dQ_n = scale sum_m dS_nm k_m,  dK_m = scale sum_n dS_nm q_n,
 * over the pairs kept by M.  Needs row AND column lists (build the mask with
 * NABLA_EMIT_COLS) and the o, lse written by nabla_attn_fwd.  Deterministic
 * (no atomics).  Workspace: nabla_workspace_size(shape, NABLA_OP_ATTN_BWD). */
int nabla_attn_bwd(const nabla_shape *shape, const nabla_params *params, const nabla_bf16 *q,
                   const nabla_bf16 *k, const nabla_bf16 *v, const nabla_bf16 *o,
                   const nabla_bf16 *dout, const float *lse, const nabla_mask *mask,
                   nabla_bf16 *dq, nabla_bf16 *dk, nabla_bf16 *dv, void *workspace,
                   size_t workspace_bytes, nabla_stream_t stream);

/* Synchronises `stream`, then returns the device-side status recorded in the
 * workspace by the last call that used it (NABLA_OK or NABLA_ERR_TIMEOUT),
 * or NABLA_ERR_CUDA if the stream reports an error. */
int nabla_status(const void *workspace, nabla_stream_t stream);

/* Static string for a status code. */
const char *nabla_strerror(int status);

#ifdef __cplusplus
}
#endif

#endif /* NABLA_H */
