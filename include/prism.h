/*
 * prism.h -- C ABI of the Prism dynamic block-sparse video self-attention
 * path for NVIDIA B200 (sm_100a).
 *
 * The path, per attention layer and head (Prism digest, "Prism：为原生 2K
 * 视频音频联合生成设计的动态稀疏注意力", overview and Fig. 2 description):
 *   prism_plan      8x8x8 macro-zones -> variation indicator g_d(m) and
 *                   density rho(m) -> block volume B(m) in {64,128,256}
 *                   -> block shape (nearest log2 candidate to l*) ->
 *                   block-contiguous permutation.
 *   prism_select    block means of Q and K -> block scores -> hybrid
 *                   Top-k U Top-p key-block sets (CSR, and its transpose).
 *   prism_attn_fwd  exact attention of every query over the tokens of its
 *                   selected key blocks; output in natural token order.
 *   prism_attn_bwd  gradients through the same selected blocks only.
 *
 * Conventions shared by every call
 *   Layout.  Batch 1.  Natural raster token order n = (t*H + y)*W + x over
 *     a T x H x W latent grid, N = T*H*W.  Q, K, V, O, dO, dQ, dK, dV are
 *     bf16 (passed as uint16_t bit patterns) laid out [N][heads][head_dim],
 *     contiguous.  The A2V norm map a2v_norm is fp32 [N].
 *   Sizes.  Z = (T/8)(H/8)(W/8) zones; NB = N/64 is the most blocks a head
 *     can have (every zone at B = 64).
 *   Memory.  Every pointer argument is DEVICE memory unless stated
 *     otherwise.  Tensor pointers (Q, K, V, O, O_res, dO, dQ, dK, dV, the
 *     bridge output of prism_a2v_norm) and the plan's block table must be
 *     16-byte aligned; a misaligned one is PRISM_ERR_INVALID_ARG.  The
 *     library cannot see a buffer's size or its device: passing buffers
 *     smaller than stated here, or on another device than the current one,
 *     is undefined (the Python binding checks both before every call).  The
 *     caller allocates and owns every buffer, including the workspaces sized
 *     by the *_workspace_size() queries; the library never allocates device
 *     memory (prism_plan_noalloc's fixed array aside).  Workspaces must be 256-byte aligned and may
 *     not be shared by calls that run concurrently.
 *   Execution.  Calls enqueue kernels on `stream` and return without waiting,
 *     except prism_select, which waits once on `stream` to read the number
 *     of selected entries (nnz).
 *   Errors.  Every call returns a prism_status.  Nothing is thrown across the
 *     ABI.  prism_last_error() returns a message for the calling thread's
 *     last failing call.  Kernels that time out on an internal wait record
 *     PRISM_ERR_TIMEOUT in the workspace; prism_workspace_status() reads it.
 */
#ifndef PRISM_H
#define PRISM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *prism_stream_t; /* the same type as cudaStream_t */

typedef enum prism_status {
  PRISM_OK = 0,
  PRISM_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad param   */
  PRISM_ERR_UNSUPPORTED = 2,  /* T/H/W not multiples of 8, head_dim not 64/128 */
  PRISM_ERR_CAPACITY = 3,     /* an output or workspace is too small          */
  PRISM_ERR_CUDA = 4,         /* a CUDA runtime call failed                   */
  PRISM_ERR_TIMEOUT = 5,      /* a kernel gave up on an internal wait         */
  PRISM_ERR_RANGE = 6         /* an attention input is infinite or NaN       */
} prism_status;

/*
 * Parameters of one layer.
 *   T, H, W        latent grid; each a positive multiple of 8 (macro-zone
 *                  edge Z_T = Z_H = Z_W = 8, Prism digest, Fig. 2 text).
 *   heads          number of attention heads (>= 1).
 *   head_dim       D, 64 or 128.
 *   tau128, tau256 density thresholds (0.5 and 0.25 on the pages, digest
 *                  section on information density).  rho >= tau128 gives
 *                  B = 64, tau256 <= rho < tau128 gives 128, else 256.
 *   eps            the small constant of g_d(m) (1e-6 here; "a tiny
 *                  constant" on the pages).
 *   topk_frac      Top-k as a kept fraction of key blocks, rounded up
 *                  (ignored when topk_abs > 0).
 *   topk_abs       Top-k as an absolute block count when > 0.
 *   top_p          Top-p threshold (0.2 on the pages' default, 0.9 in the
 *                  benchmark grids).
 *   sm_scale       attention scale; 0 selects 1/sqrt(head_dim).  The same
 *                  scale multiplies the block scores.
 *
 * Ablation variants (digest, section on the shape, guidance and sparsity
 * ablations).  Zero in all three fields is the method as published; the
 * pages' Top-k-only and Top-p-only settings need no field: top_p = 0 keeps
 * the Top-k prefix alone, and topk_frac = topk_abs = 0 (k = 1) leaves Top-p.
 *   map_exponent   a in b*_d proportional to g_d^(-a):
 *                  l*_d = -a log2 g_d + (S + a sum_d' log2 g_d')/3.  0 selects
 *                  the Lagrange value 1/2.  Any value in (0, 8].  (a = 0, the
 *                  isotropic mapping, is guidance = 3.)
 *   guidance       bit 0 drops the video term r_{v,d} from g_d, bit 1 drops
 *                  the A2V term abar*vhat_{a,d}.  guidance = 3 leaves
 *                  g_d = eps: isotropic shapes.
 *   density        what rho_raw(m) is: 0 spatial + temporal terms (the
 *                  method), 1 the spatial term only, 2 the temporal term
 *                  only, 3 the zone's A2V strength (zone mean of a2v_norm;
 *                  the heads then share rho; needs a2v_norm).
 */
typedef struct prism_params {
  int32_t T, H, W;
  int32_t heads, head_dim;
  float tau128, tau256, eps;
  float topk_frac;
  int32_t topk_abs;
  float top_p;
  float sm_scale;
  float map_exponent;
  int32_t guidance;
  int32_t density;
} prism_params;

/*
 * Output of prism_plan.  All arrays are device memory owned by the caller.
 *   zone_shape [heads][Z]     candidate id 0..15 of each zone (id order:
 *                             volume ascending, then (b_T,b_H,b_W)
 *                             lexicographic: 0 (2,4,8) ... 15 (8,8,4)).
 *   zone_g     [heads][Z][3]  g_T, g_H, g_W (float64).  May be NULL.
 *   zone_rho   [heads][Z]     normalised density rho(m) (float64). May be NULL.
 *   n_blocks   [heads]        number of blocks of each head.
 *   blocks     [heads][NB][4] per block: {p0, B, n0, shape id}: first
 *                             permuted position, volume, natural index of
 *                             the block's first (origin) token, candidate id.
 *                             Entries at index >= n_blocks[h] are unspecified.
 *   perm       [heads][N]     natural token index at permuted position p.
 *   inv_perm   [heads][N]     permuted position of natural token n.  May be
 *                             NULL.
 * Permuted order: zones in raster order (zW fastest), zone m occupying
 * positions [512m, 512m+512); blocks in raster order of the zone's block
 * grid; tokens in raster (t,y,x) order inside a block.
 */
typedef struct prism_plan_t {
  uint8_t *zone_shape;
  double *zone_g;
  double *zone_rho;
  int32_t *n_blocks;
  int32_t *blocks;
  int32_t *perm;
  int32_t *inv_perm;
} prism_plan_t;

/*
 * prism_a2v_norm -- the A2V guidance signal a = ||h_hat||_2 per video token
 * (digest, section on the zone guidance signals: the length of each video
 * position's audio-to-video cross-attention output; review, Method
 * section 1, a_{t,h,w} = ||h_hat_{t,h,w}||_2).  Run it on a layer's bridge
 * output; the next layer's prism_plan takes the result as a2v_norm.
 *   hhat      bf16 [n][ld] device rows (natural token order); only the first
 *             `width` elements of each row are read.  16-byte aligned.
 *   n         number of video tokens (rows), >= 0; 0 launches nothing.
 *   width     channels per row (the bridge output width, e.g. heads *
 *             head_dim), a positive multiple of 8, at most 2^20.
 *   ld        row stride in elements, a multiple of 8, >= width.
 *   a2v_norm  fp32 [n] device output.
 * Squares of the bf16 inputs are exact in fp32; they are summed in fp32
 * (eight partial sums per lane, then a fixed tree), deterministically, and
 * the square root is the correctly rounded sqrtf.
 * Returns PRISM_OK, PRISM_ERR_INVALID_ARG or PRISM_ERR_CUDA.
 */
int prism_a2v_norm(const uint16_t *hhat, int64_t n, int32_t width, int64_t ld, float *a2v_norm,
                   prism_stream_t stream);

/* Bytes of workspace prism_plan needs (0 on invalid params). */
size_t prism_plan_workspace_size(const prism_params *p);

/*
 * prism_plan -- zone statistics, variation indicator, density, volume,
 * shape and permutation, per head.
 *   Zone statistics: the channel variance of mean-pooled V along each axis
 *   (r_{v,d}), the A2V-norm coupling abar(m) and direction shares
 *   vhat_{a,d}(m), and rho_raw(m) = intra-zone spatial variance + temporal
 *   frame-difference variance (digest, section on zone guidance and the
 *   rho_raw equation; xyznot.com review "Prism: динамическое разреженное
 *   внимание ...", Method sections 1-2).  g_d = r_{v,d} + abar*vhat_{a,d}
 *   + eps; l*_d closed form; nearest candidate in log2 space.
 *   V         bf16 [N][heads][head_dim].
 *   a2v_norm  fp32 [N] norm of the previous layer's audio-to-video
 *             attention output per video token (prism_a2v_norm computes
 *             it), or NULL for the first layer (video guidance only).
 *             Required when p->density == 3.
 *   out       arrays to fill (see prism_plan_t).
 *   workspace, ws_bytes  at least prism_plan_workspace_size(p) bytes.
 * Returns PRISM_OK, PRISM_ERR_INVALID_ARG, PRISM_ERR_UNSUPPORTED,
 * PRISM_ERR_CAPACITY (ws_bytes too small) or PRISM_ERR_CUDA.
 */
int prism_plan(const prism_params *p, const uint16_t *V, const float *a2v_norm,
               const prism_plan_t *out, void *workspace, size_t ws_bytes,
               prism_stream_t stream);

/*
 * prism_project_v_plan -- the layer's value projection with the plan fused
 * into it: V = X Wv^T for every video token, on tcgen05 tensor cores, with
 * prism_plan's zone statistics of V computed in the GEMM's epilogue from the
 * tile just produced (the statistics come from the value features the
 * attention computes anyway: digest, section on zone guidance and Figure 4),
 * then the rest of prism_plan.  The plan never reads V back from memory; its
 * outputs are bit-identical to prism_plan(p, V, a2v_norm) on the V written
 * here (the statistics use the same arithmetic, in the same order).
 *   X         bf16 [N][C] token features, natural token order.
 *   C         channels of X: a positive multiple of 64, at most 65536.
 *   Wv        bf16 [heads*head_dim][C] projection weight (output x input, the
 *             layout of a linear layer's weight); output channel h*head_dim+d
 *             is channel d of head h.
 *   V         bf16 [N][heads][head_dim] output: X Wv^T, accumulated in fp32 and
 *             rounded to bf16.
 *   a2v_norm, out, workspace, ws_bytes  as prism_plan (the workspace size is
 *             prism_plan_workspace_size(p)).
 * X, Wv and V must be 16-byte aligned.  Returns PRISM_OK,
 * PRISM_ERR_INVALID_ARG, PRISM_ERR_UNSUPPORTED, PRISM_ERR_CAPACITY or
 * PRISM_ERR_CUDA; a kernel that gives up on an internal wait records
 * PRISM_ERR_TIMEOUT in the workspace (prism_workspace_status).
 */
int prism_project_v_plan(const prism_params *p, const uint16_t *X, int32_t C,
                         const uint16_t *Wv, uint16_t *V, const float *a2v_norm,
                         const prism_plan_t *out, void *workspace,
                         size_t ws_bytes, prism_stream_t stream);

/*
 * prism_plan_noalloc -- the same computation and outputs as prism_plan, for
 * callers that cannot allocate device memory.  Some hosts own every device
 * allocation themselves (a plugin inside another program's memory manager),
 * and some code may not pay the implicit device synchronisation of
 * cudaMalloc; neither can provide prism_plan's workspace.  This call needs
 * none: its scratch is a 4 MiB array in the library's device memory, which
 * every CUDA context that loads the library holds until the context is
 * destroyed (the runtime's primary context: until the process exits).  The
 * pages have no counterpart; it is an interface convenience.
 *   Inputs and outputs as prism_plan (the caller still passes V, a2v_norm and
 *   the arrays of `out`).
 *   Limit: grids whose scratch (heads*Z*44 bytes + Z*32 + 1 KiB, about
 *   1.8 MiB for the 2K grid with 24 heads) exceeds 4 MiB are rejected with
 *   PRISM_ERR_CAPACITY and a message; use prism_plan for those.
 *   The array exists once per CUDA context (a second context on the same
 *   device, or the primary context created again after cudaDeviceReset,
 *   has its own copy at another address).  The first call in a context
 *   looks up that context's address (cudaGetSymbolAddress, with the
 *   context current) and caches it under the context's id; make that first
 *   call before any stream capture.  All calls in one context share its
 *   array, which keeps the last call's contents (the call clears what must
 *   start at zero), so calls whose kernels overlap on the GPU race:
 *   serialise them (one stream, or events between streams).
 * Returns PRISM_OK, PRISM_ERR_INVALID_ARG, PRISM_ERR_UNSUPPORTED,
 * PRISM_ERR_CAPACITY or PRISM_ERR_CUDA.
 */
int prism_plan_noalloc(const prism_params *p, const uint16_t *V,
                       const float *a2v_norm, const prism_plan_t *out,
                       prism_stream_t stream);

/*
 * Output of prism_select.  Rows are indexed r = h*NB + i (head h, query
 * block i); rows i >= n_blocks[h] are empty.
 *   row_ptr [heads*NB + 1]  CSR offsets into col.
 *   col     [cap]           selected key-block ids, ascending in each row.
 *   cap     capacity of col (and of row) in entries (host value, in).
 *   nnz     entries written (host value, out).  When nnz > cap the call
 *           returns PRISM_ERR_CAPACITY and nnz is the capacity needed.
 *   col_ptr [heads*NB + 1]  CSC offsets (transpose), or NULL to skip it.
 *   row     [cap]           query-block ids of each key block, ascending.
 */
typedef struct prism_select_t {
  int32_t *row_ptr;
  int32_t *col;
  int64_t cap;
  int64_t nnz;
  int32_t *col_ptr;
  int32_t *row;
} prism_select_t;

/* Bytes of workspace prism_select needs (0 on invalid params). */
size_t prism_select_workspace_size(const prism_params *p);

/*
 * prism_select -- hybrid block selection (digest, section on hybrid block
 * selection; review, Method section 3): per head, block means Qbar_i and
 * Kbar_j over each block's tokens, scores s_ij = (Qbar_i . Kbar_j) * scale,
 * P_i = softmax_j(s_i), S_i = Top-k(P_i, k) U Top-p(P_i, top_p).
 * Precision: block means are fp32 running sums over the block's tokens in
 * raster order times 1/B; scores are fp32 running sums over channels of
 * separately rounded products, times the scale.  The Top-p cumulative sum
 * is exact: each weight exp(s_ij - max_j s_ij) is quantised to a multiple of
 * 2^-qb, qb = 62 - ceil(log2(nb + 1)) for a head of nb blocks (2^-48 at
 * nb = 13440, the 2K grid's maximum), and summed as 64-bit integers, so the
 * crossing does not depend on the order of the additions and the selection
 * is bit-reproducible; a sum moves by at most nb * 2^-(qb+1) of the row's
 * total.  p >= 1 keeps every block.  Order:
 * score descending, then key id ascending; "passes p" is read as ">= p"
 * with the crossing block kept.
 *   plan   output of prism_plan for the same params.
 *   Q, K   bf16 [N][heads][head_dim].
 *   out    see prism_select_t; out->nnz is written.
 * Waits once on `stream`.  Returns PRISM_OK, PRISM_ERR_INVALID_ARG,
 * PRISM_ERR_UNSUPPORTED, PRISM_ERR_CAPACITY or PRISM_ERR_CUDA.
 */
int prism_select(const prism_params *p, const prism_plan_t *plan,
                 const uint16_t *Q, const uint16_t *K, prism_select_t *out,
                 void *workspace, size_t ws_bytes, prism_stream_t stream);

/* Bytes of workspace prism_attn_fwd (backward = 0) or prism_attn_bwd
 * (backward = 1, either value of its `deterministic`; for head_dim 128 this
 * includes the fused path's fp32 dQ accumulator, 4 N heads 128 bytes) needs
 * (0 on invalid params). */
size_t prism_attn_workspace_size(const prism_params *p, int backward);

/*
 * prism_attn_fwd -- exact attention over the selected blocks (digest,
 * section on hybrid selection: full query tokens against the keys and
 * values of the selected key blocks, online softmax, no full attention
 * matrix; 64-token units, training section).  For every query token q of
 * block i:  O_q = sum_k softmax_k(q.k * scale) v_k  over the tokens k of
 * the blocks in S_i;  lse_q = log sum_k exp(q.k * scale).
 *   Q, K, V   bf16 [N][heads][head_dim].
 *   O         bf16 [N][heads][head_dim], natural order (inverse permutation
 *             applied).
 *   O_res     bf16 [N][heads][head_dim] or NULL: the rounding residual
 *             O_fp32 - O (rounded to bf16), so that O + O_res carries the
 *             fp32 accumulator to ~2^-17 relative.  prism_attn_bwd uses it
 *             for Delta = rowsum(dO * O); without it Delta is formed from the
 *             bf16 O, whose rounding dominates the gradient error of rows
 *             with sharp attention.
 *   lse       fp32 [heads][N], natural order (natural log).
 * Runs on tcgen05 tensor cores with fp32 accumulation.  The operands are
 * fp16: Q, K, V convert from bf16 exactly for 2^-17 <= |x| <= 65504 and for
 * 0, and within 2^-25 below that.  A head whose Q, K or V holds a value
 * above 65504 (any finite bf16 value is accepted) is converted with a
 * power-of-two pre-scale that the kernels fold back exactly into the score
 * scale and the output; heads within the fp16 range are unaffected.  An
 * infinite or NaN input records PRISM_ERR_RANGE in the workspace.  The
 * probabilities P (in [0, 256] under the lazy rescaling) are rounded to fp16,
 * 8x finer than bf16.
 * Returns PRISM_OK, PRISM_ERR_INVALID_ARG, PRISM_ERR_UNSUPPORTED,
 * PRISM_ERR_CAPACITY or PRISM_ERR_CUDA.
 */
int prism_attn_fwd(const prism_params *p, const prism_plan_t *plan,
                   const prism_select_t *sel, const uint16_t *Q,
                   const uint16_t *K, const uint16_t *V, uint16_t *O,
                   uint16_t *O_res, float *lse, void *workspace,
                   size_t ws_bytes, prism_stream_t stream);

/*
 * prism_attn_bwd -- gradients of prism_attn_fwd through the selected blocks
 * only; the plan and the selection are constants (digest, training section).
 *   O, lse    outputs of prism_attn_fwd for the same inputs.
 *   O_res     the forward's O_res, or NULL (Delta from the bf16 O alone).
 *   dO        bf16 [N][heads][head_dim] upstream gradient.
 *   dQ,dK,dV  [N][heads][head_dim]; bf16 when grad_fp32 == 0, fp32 else.
 *   deterministic  0: for head_dim 128, one kernel per 128-key tile forms
 *             dK, dV and that tile's share of dQ (dQ = scale dS K added into
 *             an fp32 accumulator in the workspace by fp32 reductions, then
 *             converted to dQ); 10 P D flops for P computed query-key pairs.
 *             The order of those adds varies from run to run, so dQ may
 *             differ in its last bits between runs (dK, dV do not).
 *             1 (and head_dim 64 always): two kernels, one per 128-key tile
 *             for dK, dV and one per 128-query tile for dQ, which computes
 *             S and dP a second time (14 P D flops); every output is
 *             bitwise reproducible.  Any other value is PRISM_ERR_INVALID_ARG.
 * sel must carry the transpose (col_ptr/row non-NULL).
 * Returns PRISM_OK, PRISM_ERR_INVALID_ARG, PRISM_ERR_UNSUPPORTED,
 * PRISM_ERR_CAPACITY or PRISM_ERR_CUDA.
 */
int prism_attn_bwd(const prism_params *p, const prism_plan_t *plan,
                   const prism_select_t *sel, const uint16_t *Q,
                   const uint16_t *K, const uint16_t *V, const uint16_t *O,
                   const uint16_t *O_res, const uint16_t *dO,
                   const float *lse, void *dQ, void *dK, void *dV,
                   int grad_fp32, int deterministic, void *workspace,
                   size_t ws_bytes, prism_stream_t stream);

/* Waits on `stream` and returns the status a kernel recorded in
 * `workspace`: PRISM_OK, PRISM_ERR_TIMEOUT, PRISM_ERR_RANGE (an attention
 * call met an infinite or NaN Q/K/V/dO value), PRISM_ERR_UNSUPPORTED (the
 * fused backward found its shared-memory window not 1024-byte aligned; its
 * layout fills the window and cannot realign it), or PRISM_ERR_CUDA. */
int prism_workspace_status(const void *workspace, prism_stream_t stream);

/* Message of the calling thread's last failing call ("" if none).  The
 * string is owned by the library and valid until the thread's next call. */
const char *prism_last_error(void);

/* Number of kernels this process has launched through the library so far
 * (host-side counter, incremented at every launch; never reset). */
uint64_t prism_kernel_launches(void);

/* Optional timing of the library's kernels, for measurement (not meant to be
 * toggled by one thread while another launches through the library).  When
 * enabled, every kernel launch of the path is bracketed by a CUDA event pair
 * recorded on its launching stream.
 * prism_kernel_timing(1) clears the records and enables; (0) clears and
 * disables.  Returns PRISM_OK. */
int prism_kernel_timing(int enable);

/* Number of kernel timing ids.  Ids, in order: 0 zone_video_stats,
 * 1 block_mean, 2 block_score, 3 select_row, 4 attn_fwd, 5 attn_bwd_dkdv,
 * 6 attn_bwd_dq, 7 a2v_norm, 8 zone_a2v_stats, 9 plan_finalize, 10 perm,
 * 11 select_scan, 12 csr_fill, 13 csc_count, 14 csc_scan, 15 csc_fill,
 * 16 csc_sort, 17 permute3, 18 unit_block, 19 tile_units, 20 bwd_prep,
 * 21 project_v, 22 range_fix (both launches of the pre-scale fix-up of
 * operands above the fp16 range; their blocks return at once when no value
 * is), 23 attn_bwd_fused (dK, dV and dQ in one kernel), 24 dq_convert
 * (the fused kernel's fp32 dQ accumulator to the natural-order output). */
#define PRISM_KERNEL_TIMING_IDS 25

/* Reads the records of kernel `id` (0 .. PRISM_KERNEL_TIMING_IDS - 1): waits
 * for its events, and returns the number of timed launches, their total
 * milliseconds and the kernel's name (library-owned string).  Returns
 * PRISM_OK, PRISM_ERR_INVALID_ARG (id out of range) or PRISM_ERR_CUDA. */
int prism_kernel_timing_read(int id, int *launches, double *total_ms,
                             const char **name);

/* Library version, "major.minor.patch". */
const char *prism_version(void);

/*
 * prism_diag_exp2 -- diagnostics.  Evaluates, for n fp32 inputs x (device
 * memory), two ways of forming softmax weights: y_poly = 2^x from the
 * library's FMA-pipe polynomial (x clamped to [-125, 64]; relative error at
 * most 7.5e-5, below half an fp16 ulp) and y_mufu = 2^x from the MUFU
 * instruction.  The attention kernels can move a share of their
 * exponentials to the polynomial; they currently use MUFU for all of them,
 * which measured faster.  Outputs are fp32 device arrays of n entries.
 * Returns PRISM_OK, PRISM_ERR_INVALID_ARG or PRISM_ERR_CUDA.
 */
int prism_diag_exp2(const float *x, float *y_poly, float *y_mufu, int64_t n, prism_stream_t stream);

/*
 * prism_diag_wait_timeout -- diagnostics: exercises the failure path of the
 * kernels' bounded waits without any fault.  Clears the workspace header,
 * then runs one warp that waits on an mbarrier nothing completes; after
 * limit_cycles SM cycles (at most 1e9) it gives up and records
 * PRISM_ERR_TIMEOUT in the workspace status word, as any library kernel does
 * when one of its waits runs out.  prism_workspace_status(workspace) then
 * returns PRISM_ERR_TIMEOUT, and the context stays usable.
 *   workspace  device memory of at least 256 bytes, 256-byte aligned.
 * Returns PRISM_OK (the kernel was enqueued), PRISM_ERR_INVALID_ARG or
 * PRISM_ERR_CUDA.
 */
int prism_diag_wait_timeout(void *workspace, size_t ws_bytes, int64_t limit_cycles, prism_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_H */
