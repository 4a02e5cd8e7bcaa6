/*
 * salad.h - C ABI of libsalad, a B200 (sm_100a) implementation of the SALAD
 * hybrid attention layer of a video diffusion transformer:
 *
 *   out = SparseAttn_STSWA(q, k, v) + g[b,h] * ( LinAttn_ReLU(q, k, v) . W )
 *
 * Sources, all on the SALAD pages: the parallel sparse + linear branches that
 * share Q/K/V (SALAD technical summary, section 2.1 "Architecture design";
 * sciencestack abstract and Figure 3, the SALAD module overview);
 * ST-SWA static sparsity (sciencestack Figure 1; summary section 5); ReLU
 * linear attention of O(N) cost (summary section 2.1); the learnable projection
 * that down-weights the linear output (summary section 2.2, LWSS); the
 * scalar gate in (0,1) that depends on the input (summary section 2.2, ITADS;
 * sciencestack TL;DR); dropping the linear branch when its gate is negligible
 * (summary section 2.3).
 *
 * Conventions shared by every call:
 *   - Token n of a T x H x W latent grid is (t, y, x) with n = (t*H + y)*W + x.
 *   - Tensors q, k, v, out are bf16, contiguous [B][N][Hh][d] (head-interleaved,
 *     as a DiT's fused QKV projection writes them).
 *   - Block I holds tokens [I*block, min(N, (I+1)*block)); nb = ceil(N/block).
 *   - All device pointers are caller-owned; the library never allocates device
 *     memory and keeps no state between calls apart from cached driver entry
 *     points.  Calls are asynchronous on `stream` unless stated otherwise.
 *   - Every entry point returns a salad_status; argument errors are detected on
 *     the host before anything is launched.
 */
#ifndef SALAD_H_
#define SALAD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* salad_stream_t;

typedef enum {
  SALAD_OK = 0,
  SALAD_ERR_INVALID_ARG = -1,    /* null/misaligned pointer, bad size or window */
  SALAD_ERR_UNSUPPORTED = -2,    /* valid but not built: d or block not in {64,128}, ... */
  SALAD_ERR_CAPACITY = -3,       /* col_idx too small for the mask (see nnz_out) */
  SALAD_ERR_WORKSPACE = -4,      /* workspace smaller than salad_workspace_bytes() */
  SALAD_ERR_CUDA = -5,           /* a CUDA runtime/driver call or launch failed */
  SALAD_ERR_DEVICE_TIMEOUT = -6, /* a kernel gave up waiting (see salad_check_status) */
  SALAD_ERR_OUT_OF_MEMORY = -7,  /* the device had no memory left for the static scratch */
  SALAD_ERR_BAD_MASK = -8        /* checking build (SALAD_DEBUG): a kernel skipped a malformed mask row */
} salad_status;

/*
 * Number of blocks nb = ceil(T*H*W / block).  Host only.
 * Errors: INVALID_ARG for non-positive sizes, N >= 2^31 or nb == NULL.
 */
int salad_mask_num_blocks(int T, int H, int W, int block, int* nb);

/*
 * Static spatio-temporal sliding-window block mask (ST-SWA: sciencestack
 * Figure 1; the SPADE page's 3-D grid of video blocks describes the same
 * T x H x W block structure).  For every head h and query block I it lists, in
 * ascending order, the key blocks J for which SOME real token pair i in I,
 * j in J satisfies |t_i - t_j| <= wt, |y_i - y_j| <= wh, |x_i - x_j| <= ww.
 *
 *   windows   HOST int32 [num_heads][3] = (wt, wh, ww), inclusive half-widths,
 *             each >= 0.
 *   row_ptr   DEVICE int32 [num_heads*nb + 1]: row (h, I) is
 *             col_idx[row_ptr[h*nb+I] .. row_ptr[h*nb+I+1]); offsets are global.
 *   col_idx   DEVICE int32 [col_capacity]; may be NULL when col_capacity == 0.
 *   nnz_out   HOST, nullable: receives the total number of kept pairs.
 * The call synchronises `stream` once (to read the count) and is meant to run
 * once per (grid, block, windows), outside any timed or captured region.
 * Errors: INVALID_ARG (sizes, negative window, null row_ptr, num_heads outside
 * [1, 256]); CAPACITY when col_capacity < nnz (row_ptr is then complete,
 * col_idx untouched, *nnz_out set); CUDA.
 */
int salad_build_block_mask(int T, int H, int W, int block, int num_heads, const int32_t* windows,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int64_t* nnz_out,
                           salad_stream_t stream);

/*
 * 3-D tile blocks (the SPADE page's 3-D grid of video blocks; the SALAD
 * summary's block structure over the T x H x W latent): block I is the box of
 * bt x bh x bw grid points
 *   t in [ti*bt, ti*bt+bt),  y in [yi*bh, yi*bh+bh),  x in [xi*bw, xi*bw+bw)
 * with boxes numbered in raster order, I = (ti*nh + yi)*nw + xi, nh =
 * ceil(H/bh), nw = ceil(W/bw).  bt must divide T; boxes at the bottom and right
 * edges may stick out of the grid, and their slots outside it hold no token.
 * Slot s = (tt*bh + yy)*bw + xx of box I holds token (t*H + y)*W + x of the
 * flat [T][H][W] sequence.
 * salad_tile_num_blocks: nb = (T/bt) * nh * nw.  Host only.  Errors:
 * INVALID_ARG (non-positive sizes, T*H*W >= 2^31, nb == NULL); UNSUPPORTED
 * when bt does not divide T.
 */
int salad_tile_num_blocks(int T, int H, int W, int bt, int bh, int bw, int* nb);

/*
 * The ST-SWA window mask over 3-D tile blocks: row (h, I) lists, in ascending
 * order, the boxes J holding SOME token pair i in I, j in J within the head's
 * windows (|t_i - t_j| <= wt, |y_i - y_j| <= wh, |x_i - x_j| <= ww).  Since each
 * box covers a product of ranges (clipped to the grid), that is: on every axis
 * the gap between the two boxes' ranges is within that axis' window.
 * Arguments, layouts, synchronisation and errors as salad_build_block_mask
 * (nb from salad_tile_num_blocks; UNSUPPORTED when bt does not divide T).
 */
int salad_build_tile_mask(int T, int H, int W, int bt, int bh, int bw, int num_heads, const int32_t* windows,
                          int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int64_t* nnz_out,
                          salad_stream_t stream);

/*
 * Host-side check of a block mask in the CSR layout the layer takes (for masks
 * a caller builds or transposes itself): row_ptr[0] == 0, row_ptr
 * non-decreasing with at most nb entries a row, every column in [0, nb) and the
 * columns of a row strictly ascending.
 *   row_ptr  HOST int32 [rows + 1];  col_idx HOST int32 [row_ptr[rows]] (may be
 *            NULL when every row is empty).
 *   bad_row  HOST, nullable: the first offending row (-1 when the mask is valid).
 * Returns SALAD_OK or SALAD_ERR_INVALID_ARG.  Reads host memory only.
 */
int salad_validate_mask(const int32_t* row_ptr, const int32_t* col_idx, int64_t rows, int nb, int64_t* bad_row);

/*
 * Bytes of device workspace salad_attn_forward needs for these sizes (0 on bad
 * arguments).  The workspace holds a status word, the linear-branch state
 * [S | z] of every (b, h) and the split-N partial sums.  It must be zero-filled
 * once after allocation (the status word must start at 0); calls leave it
 * reusable.  One workspace must not be shared by calls that may overlap.
 */
size_t salad_workspace_bytes(int B, int N, int num_heads, int d);

/*
 * The SALAD layer forward (sciencestack abstract and Figure 3; summary
 * sections 2.1-2.3):
 *   o_sp_i  = sum_{j in K(i)} softmax_j(scale * q_i . k_j) v_j, where K(i) is
 *             every real token of the key blocks kept for i's query block
 *   S, z    = sum_j relu(k_j) v_j^T (d x d),  sum_j relu(k_j)   over all N
 *   o_lin_i = relu(q_i)^T S / (relu(q_i) . z + eps)
 *   out_i   = o_sp_i + g[b,h] * (o_lin_i W)      (y_e = sum_c o_lin_c W[c][e])
 * When g[b,h] == 0 the linear branch of (b, h) is skipped entirely and
 * out_i = o_sp_i exactly (branch dropping).
 *
 *   q, k, v      DEVICE bf16 [B][N][Hh][d], 16-byte aligned.
 *   d            64 or 128.   block: 64 or 128.   Hh*d*2 bytes % 16 == 0.
 *   row_ptr, col_idx  DEVICE, from salad_build_block_mask with the same N
 *                (= T*H*W), block and num_heads; columns ascending.  (That
 *                builder keeps every diagonal block; a row left empty by other
 *                means gives those queries no sparse term: out = g * y.)
 *   w_proj       DEVICE bf16 [d][d] (row c, column e), 16-byte aligned.
 *   gate         DEVICE fp32 [B][Hh].
 *   softmax_scale  <= 0 selects 1/sqrt(d).   eps: added to the denominator.
 *   out          DEVICE bf16 [B][N][Hh][d], 16-byte aligned; may not alias q/k/v.
 *   workspace    DEVICE, >= salad_workspace_bytes(B, N, Hh, d), 256-byte aligned.
 * Never synchronises.  Arithmetic: bf16 tensor-core products with fp32
 * accumulation, fp32 softmax, one round-to-nearest-even to bf16 at the store.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA (launch failures).  A
 * device-side time-out is reported later by salad_check_status.
 */
int salad_attn_forward(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d,
                       int block, const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj,
                       const float* gate, float softmax_scale, float eps, void* out, void* workspace,
                       size_t workspace_bytes, salad_stream_t stream);

/*
 * salad_attn_forward (mask rows per head, or per (b, h) when mask_per_bh != 0)
 * that also writes what a training forward keeps for the backward pass:
 *   lse[b][h][i] = log sum_{j in K(i)} exp(scale * q_i . k_j)   (natural log;
 *                  -inf for a row whose blocks keep no key)
 *   lse   DEVICE fp32 [B][Hh][N], 4-byte aligned.
 * Everything else as salad_attn_forward.  fp32: the row maximum the kernel
 * keeps plus log2 of its fp32 row sum, times ln 2.
 */
int salad_attn_forward_lse(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d,
                           int block, const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj,
                           const float* gate, float softmax_scale, float eps, int mask_per_bh, void* out, float* lse,
                           void* workspace, size_t workspace_bytes, salad_stream_t stream);

/*
 * Backward pass of the sparse branch (block-sparse softmax attention over the
 * kept key blocks), for training through the layer (the SALAD summary,
 * section 3, fine-tunes the model with the layer in place).  With
 * p_ij = exp(scale q_i.k_j - lse_i) over the kept keys of i and o_i the branch
 * output (out of salad_attn_forward_lse when every gate is 0):
 *   D_i = dout_i . o_i,   ds_ij = p_ij (dout_i . v_j - D_i)
 *   dq_i = scale sum_j ds_ij k_j,  dk_j = scale sum_i ds_ij q_i,  dv_j = sum_i p_ij dout_i
 *   q, k, v, o, dout  DEVICE bf16 [B][N][Hh][d], 16-byte aligned; d = 64 or 128.
 *   lse        DEVICE fp32 [B][Hh][N] from salad_attn_forward_lse (natural log).
 *   block      128 (raster blocks).
 *   row_ptr, col_idx      the mask the forward used (rows per head, or per
 *                         (b, h) when mask_per_bh != 0).
 *   t_row_ptr, t_col_idx  its transpose with the same row numbering: row
 *                         (h or b*Hh+h, J) lists, ascending, the query blocks
 *                         whose rows keep key block J.  The window masks of
 *                         salad_build_block_mask are symmetric: pass the same
 *                         arrays.
 *   softmax_scale  <= 0 selects 1/sqrt(d) (as in the forward).
 *   dq, dk, dv DEVICE fp32 [B][N][Hh][d], 16-byte aligned.
 *   workspace  DEVICE, >= salad_backward_workspace_bytes(B, N, Hh), 256-byte
 *              aligned; its first word is a status word like the forward's
 *              (zero it once after allocation; read it with salad_check_status).
 * Arithmetic: bf16 tensor-core products with fp32 accumulation (P and dS are
 * rounded to bf16 as operands), fp32 elsewhere.  Never synchronises.
 * Errors: INVALID_ARG, UNSUPPORTED (d, block), WORKSPACE, CUDA.
 */
/*
 * salad_attn_forward on inputs and output in HOST memory, for a caller whose
 * tensors live on the host: the host-to-device copies of one chunk of heads
 * run while the chunk before it computes and the one before that copies its
 * output back.  The layer's (b, h) units are independent (SALAD summary section
 * 2.1: every head has its own mask rows, linear-branch state and output), so a
 * chunk (one batch element, heads [h0, h0 + heads_per_chunk)) is a complete
 * forward of its own (salad_attn_forward_heads on it).
 *   q_host, k_host, v_host  HOST bf16 [B][N][Hh][d], read; out_host HOST bf16
 *                  [B][N][Hh][d], written.  Page-locked memory (cudaHostAlloc
 *                  or cudaHostRegister) for the copies to overlap; pageable
 *                  memory works but serialises them.
 *   q_dev, k_dev, v_dev, out_dev  DEVICE bf16 [B][N][Hh][d], 16-byte aligned:
 *                  the staging copies (they hold the inputs and the output
 *                  afterwards).  The library allocates nothing.
 *   row_ptr, col_idx, w_proj, gate  DEVICE, as salad_attn_forward (a per-head
 *                  raster mask from salad_build_block_mask).
 *   heads_per_chunk  > 0, or 0 for about six chunks per batch element (at 12
 *                  heads, 32,760 tokens: 6.43 ms per call against 5.45 ms for
 *                  the input copies alone and 8.2 ms with one chunk).
 *   workspace      >= salad_workspace_bytes(1, N, heads_per_chunk, d) (chunks
 *                  run one after another on `stream` and share it).
 *   stream         the forwards; copy_in, copy_out  two other streams for the
 *                  copies.  The copies wait for the work queued on `stream`
 *                  before the call, and `stream` waits for the last output copy:
 *                  synchronising `stream` (or an event recorded on it after the
 *                  call) covers the whole call.
 * Arithmetic, rounding and results as salad_attn_forward_heads per chunk.
 * Errors: INVALID_ARG (null, misaligned device buffers, equal streams),
 * UNSUPPORTED (block, d, Hh > 65535), WORKSPACE, CUDA; otherwise as
 * salad_attn_forward.
 */
int salad_attn_forward_host(const void* q_host, const void* k_host, const void* v_host, void* out_host, int B,
                            int N, int num_heads, int d, int block, const int32_t* row_ptr, const int32_t* col_idx,
                            const void* w_proj, const float* gate, float softmax_scale, float eps,
                            int heads_per_chunk, void* q_dev, void* k_dev, void* v_dev, void* out_dev,
                            void* workspace, size_t workspace_bytes, salad_stream_t stream,
                            salad_stream_t copy_in, salad_stream_t copy_out);

size_t salad_backward_workspace_bytes(int B, int N, int num_heads);
int salad_attn_backward_sparse(const void* q, const void* k, const void* v, const void* o, const void* dout,
                               const float* lse, int B, int N, int num_heads, int d, int block,
                               const int32_t* row_ptr, const int32_t* col_idx, const int32_t* t_row_ptr,
                               const int32_t* t_col_idx, int mask_per_bh, float softmax_scale, float* dq, float* dk,
                               float* dv, void* workspace, size_t workspace_bytes, salad_stream_t stream);

/*
 * Backward pass of the whole layer: the sparse branch as above plus the linear
 * branch, its projection and the gate (the gradients the fine-tuning needs).
 * With a_i = relu(q_i), S and z the branch's state, den_i = a_i.z + eps,
 * o_i = a_i^T S / den_i, y_i = o_i W, out_i = o_sp_i + g y_i:
 *   dgate[b][h] = sum_i dout_i.y_i;   dW = sum over (b, h, i) of o_i^T (g dout_i)
 *   du_i = (g dout_i W^T) / den_i,  dden_i = -(g dout_i W^T).o_i / den_i,
 *   dS = sum_i a_i du_i^T,  dz = sum_i dden_i a_i
 *   dq_i += [q_i > 0] (S du_i + dden_i z),  dk_j += [k_j > 0] (dS v_j + dz),
 *   dv_j += dS^T relu(k_j)
 * and the sparse branch's gradients with o_sp_i = out_i - g y_i in D_i.
 *   out, lse   from salad_attn_forward_lse with the same inputs.
 *   w_proj     DEVICE bf16 [d][d], 16-byte aligned;  gate DEVICE fp32 [B][Hh].
 *   dq, dk, dv DEVICE fp32 [B][N][Hh][d], 16-byte aligned (written).
 *   dw         DEVICE fp32 [d][d];  dgate DEVICE fp32 [B][Hh] (written).
 *   workspace  DEVICE, >= salad_layer_backward_workspace_bytes(B, N, Hh, d),
 *              256-byte aligned, status word first (zero it once).
 * Other arguments as salad_attn_backward_sparse.  The linear branch runs on the
 * tensor cores through T = S W: a_i T and dout_i T^T per row, M = sum_i a_i^T
 * (g / den_i) dout_i over the rows, dS = M W^T and dW = sum over (b, h) of S^T M;
 * every operand that is not already bf16 (T, (g / den_i) dout_i, dS) enters as
 * bf16 hi + lo halves, accumulation is fp32 and every sum runs in a fixed order
 * (deterministic).  The workspace is O(B Hh (N + d^2)), about 40 MB for
 * 32,760 tokens x 12 heads of d = 128.  Errors: INVALID_ARG, UNSUPPORTED (d,
 * block != 128, B*Hh > 65535), WORKSPACE, CUDA; a stalled wait sets the status
 * word's time-out bit (salad_check_status).
 */
size_t salad_layer_backward_workspace_bytes(int B, int N, int num_heads, int d);
int salad_attn_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                        const float* lse, int B, int N, int num_heads, int d, int block, const int32_t* row_ptr,
                        const int32_t* col_idx, const int32_t* t_row_ptr, const int32_t* t_col_idx, int mask_per_bh,
                        const void* w_proj, const float* gate, float softmax_scale, float eps, float* dq, float* dk,
                        float* dv, float* dw, float* dgate, void* workspace, size_t workspace_bytes,
                        salad_stream_t stream);

/*
 * Top-K dynamic block mask.  The SALAD summary (section 5) says the method also
 * applies to Top-K dynamic sparse attention and gives no scoring rule; the rule
 * implemented here is a reading of that sentence:
 *   qm[b][h][I] = mean of q[b][i][h][:] over the real tokens i of block I,
 *   km[b][h][J] likewise for k,  score(I, J) = qm[b][h][I] . km[b][h][J],
 *   row (b, h, I) keeps the kk = min(keep, nb) key blocks J with the highest
 *   scores (equal scores: the smaller J first), listed in ascending J.
 * The arithmetic is fixed so that the result is reproducible bit for bit: fp32
 * sums over the block's tokens in token order, one fp32 division by the token
 * count, and each score a chain of fused multiply-adds over the features in
 * order, starting from 0.
 *
 *   q, k       DEVICE bf16 [B][N][Hh][d], 4-byte aligned, d = 64 or 128.   block >= 1,
 *              nb <= 2048.
 *   keep       >= 1 (clamped to nb).
 *   row_ptr    DEVICE int32 [B*Hh*nb + 1]: row r = (b*Hh + h)*nb + I holds
 *              col_idx[r*kk .. (r+1)*kk).   col_idx: DEVICE int32 [B*Hh*nb*kk].
 *   workspace  DEVICE, >= salad_topk_workspace_bytes(B, N, Hh, d, block), 4-byte
 *              aligned (the block means).
 * Rows are per (b, h): pass the mask to salad_attn_forward_bh.  Never
 * synchronises.  Errors: INVALID_ARG, UNSUPPORTED (d, nb > 2048, B*Hh > 65535, sizes),
 * WORKSPACE, CUDA.
 */
/*
 * The SALAD layer forward over 3-D tile blocks (salad_tile_num_blocks): the
 * same output as salad_attn_forward, token by token, with the sparse branch's
 * key set K(i) = every real token of the boxes kept for the box holding i.
 *   q, k, v, out  DEVICE bf16 [B][T][H][W][Hh][d] (the [B][N][Hh][d] layout
 *                 with N = T*H*W in raster order), 16-byte aligned.
 *   bt*bh*bw      must be 128 (one box fills one 128-row query tile); T % bt == 0.
 *   row_ptr, col_idx  DEVICE, from salad_build_tile_mask with the same grid,
 *                 tile and num_heads.
 *   Other arguments, workspace (salad_workspace_bytes(B, T*H*W, Hh, d)),
 *   arithmetic and errors as salad_attn_forward; UNSUPPORTED when
 *   bt*bh*bw != 128 or bt does not divide T.
 */
int salad_attn_forward_tiles(const void* q, const void* k, const void* v, int B, int T, int H, int W, int bt,
                             int bh, int bw, int num_heads, int d, const int32_t* row_ptr, const int32_t* col_idx,
                             const void* w_proj, const float* gate, float softmax_scale, float eps, void* out,
                             void* workspace, size_t workspace_bytes, salad_stream_t stream);

/*
 * The dynamic gate of the linear branch and branch dropping.  The SALAD
 * summary (section 2.2, ITADS) has a lightweight module turn the denoising
 * timestep and the hidden state into a global factor s in (0, 1) through a
 * sigmoid, and (section 2.3) drops the linear branch at inference where s is
 * very low.  The module is not given; the one implemented here is the plainest
 * reading, one affine map per head over the timestep embedding and the token
 * mean of the layer's queries (the hidden state the layer sees):
 *   s[b][h]    = sigmoid(w_t[h] . t_emb[b] + w_x[h] . (1/N) sum_n q[b][n][h][:] + beta[h])
 *   gate[b][h] = 0 if s[b][h] < threshold (salad_attn_forward then skips the
 *                linear branch of (b, h) entirely), s[b][h] otherwise.
 * fp32 arithmetic in a fixed order (per feature: within a run of tokens, four
 * interleaved token streams summed in token order and added in stream order;
 * the runs' sums in eight interleaved groups added in order; fixed tree sums
 * for the dot products), so repeated calls give the same bits.
 *
 *   q          DEVICE bf16 [B][N][Hh][d], 16-byte aligned; d = 64 or 128.
 *   t_emb      DEVICE fp32 [B][E];  w_t DEVICE fp32 [Hh][E] (both may be NULL
 *              when E == 0).   w_x DEVICE fp32 [Hh][d].   beta DEVICE fp32 [Hh].
 *   threshold  finite; <= 0 drops nothing, > 1 drops every branch.
 *   s_out      DEVICE fp32 [B][Hh] or NULL: s before dropping.
 *   gate_out   DEVICE fp32 [B][Hh]: the gate salad_attn_forward takes.
 *   workspace  DEVICE, >= salad_gate_workspace_bytes(B, N, Hh, d), 16-byte
 *              aligned; no initialisation needed.
 * Never synchronises.  Errors: INVALID_ARG, UNSUPPORTED (d, B > 65535),
 * WORKSPACE, CUDA.
 */
size_t salad_gate_workspace_bytes(int B, int N, int num_heads, int d);
int salad_gate_forward(const void* q, int B, int N, int num_heads, int d, const float* t_emb, int E,
                       const float* w_t, const float* w_x, const float* beta, float threshold, float* s_out,
                       float* gate_out, void* workspace, size_t workspace_bytes, salad_stream_t stream);

size_t salad_topk_workspace_bytes(int B, int N, int num_heads, int d, int block);
int salad_build_topk_mask(const void* q, const void* k, int B, int N, int num_heads, int d, int block, int keep,
                          int32_t* row_ptr, int32_t* col_idx, void* workspace, size_t workspace_bytes,
                          salad_stream_t stream);

/*
 * salad_attn_forward with a mask whose rows are per (b, h) — row (b*Hh + h)*nb
 * + I lists the key blocks of query block I of batch element b, head h (as
 * salad_build_topk_mask writes them) — instead of per head.  Same arguments,
 * rules and errors otherwise.
 */
int salad_attn_forward_bh(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d,
                          int block, const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj,
                          const float* gate, float softmax_scale, float eps, void* out, void* workspace,
                          size_t workspace_bytes, salad_stream_t stream);

/*
 * The transpose of a block mask, for the backward pass (its dk and dv walk
 * the query blocks that keep a key block).  For every group g (a head, or a
 * (b, h) for a mask with rows per (b, h)) and key block J, t_col_idx lists in
 * ascending order the query blocks I whose row (g, I) keeps J.
 *   row_ptr, col_idx  DEVICE, groups*nb rows with ascending columns (as the mask
 *                     builders write them).
 *   t_row_ptr         DEVICE int32 [groups*nb + 1], written.
 *   t_col_idx         DEVICE int32 [nnz], nnz = row_ptr[groups*nb] (a
 *                     transpose keeps every pair), written.
 * Asynchronous on `stream`; deterministic.  The window masks are symmetric and
 * are their own transpose.  Errors: INVALID_ARG (null, misaligned, non-positive
 * sizes), UNSUPPORTED (groups > 65535 or groups*nb*nb >= 2^31), CUDA.
 */
int salad_transpose_block_mask(const int32_t* row_ptr, const int32_t* col_idx, int groups, int nb,
                               int32_t* t_row_ptr, int32_t* t_col_idx, salad_stream_t stream);

/*
 * salad_attn_forward on a range of heads: q, k, v and out are full
 * [B][N][heads_total][d] tensors, and the call reads and writes heads
 * [head_begin, head_begin + head_count) of them only.  The layer's (b, h) units
 * are independent (every head has its own mask rows, linear-branch state and
 * output; SALAD summary section 2.1), so a head-parallel job runs one range per
 * GPU with no exchange in the forward pass; the other heads of out are left
 * untouched.
 *   row_ptr, col_idx  the mask of the range's heads (head_count rows of blocks,
 *                     as salad_build_block_mask builds it from their windows).
 *   gate              DEVICE fp32 [B][head_count]: the range's gates.
 *   workspace         >= salad_workspace_bytes(B, N, head_count, d).
 * Everything else as salad_attn_forward (d, block, alignment, eps, stream).
 * Errors: INVALID_ARG also when the range does not lie inside [0, heads_total);
 * UNSUPPORTED when heads_total > 65535; otherwise as salad_attn_forward.
 */
int salad_attn_forward_heads(const void* q, const void* k, const void* v, int B, int N, int heads_total,
                             int head_begin, int head_count, int d, int block, const int32_t* row_ptr,
                             const int32_t* col_idx, const void* w_proj, const float* gate, float softmax_scale,
                             float eps, void* out, void* workspace, size_t workspace_bytes, salad_stream_t stream);

/* Size of the static device scratch behind salad_attn_forward_static: 32 MiB.
 * The scratch grows with B*Hh, not with N (salad_workspace_bytes): for any N it
 * covers B*Hh <= 254 at d = 128 and B*Hh <= 1008 at d = 64.  The 12-head
 * 32,760-token layer needs 20 MB, the 40-head 75,600-token one 21 MB. */
#define SALAD_STATIC_SCRATCH_BYTES (32u << 20)

/*
 * salad_attn_forward for callers that cannot allocate device memory.  (The
 * SALAD pages have no counterpart of this entry point; it changes how the
 * scratch is provided, not what is computed.)
 *
 * Some callers cannot call cudaMalloc: a plugin inside a serving engine that
 * reserves the device memory pool up front and forbids other allocations, or a
 * latency-critical path that may not pay cudaMalloc's implicit device
 * synchronisation.  This entry point takes the same arguments as
 * salad_attn_forward minus the workspace: its scratch is a file-scope static
 * device array of SALAD_STATIC_SCRATCH_BYTES that every GPU loading the
 * library holds until the process exits.  It calls no cudaMalloc, cudaFree or
 * allocating library routine.
 *   - Each call asks the runtime for the array's device address on the
 *     current device.  The first call on a device loads the library's device
 *     code there, and with it the driver maps the 32 MiB array: make that first
 *     call before any stream capture, and before the engine reserves its memory
 *     pool.  If the device has no memory left for the array the call returns
 *     SALAD_ERR_OUT_OF_MEMORY.  After a context reset (cudaDeviceReset) the next
 *     call maps the array again, in the new context.
 *   - Every call shares the one array, which keeps the previous call's
 *     contents.  Calls that may overlap on the GPU (other streams, other
 *     threads) race on the array: serialise them.
 *   - A device time-out is recorded in the array's status word and stays there
 *     until salad_check_status_static reads and clears it; an output produced
 *     by a call that timed out is invalid.
 * Errors: as salad_attn_forward; WORKSPACE when salad_workspace_bytes(B, N,
 * num_heads, d) exceeds SALAD_STATIC_SCRATCH_BYTES; OUT_OF_MEMORY as above;
 * CUDA when the scratch address cannot be obtained.
 */
int salad_attn_forward_static(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d,
                              int block, const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj,
                              const float* gate, float softmax_scale, float eps, void* out, salad_stream_t stream);

/*
 * salad_check_status for salad_attn_forward_static, whose status word lives in
 * the static scratch of the current device: synchronises `stream`, then reads
 * and clears that word.  Returns SALAD_ERR_DEVICE_TIMEOUT if a kernel of an
 * earlier static call on this device gave up on a bounded wait, SALAD_ERR_CUDA
 * if the stream reports an error, SALAD_OK otherwise.  (No counterpart on the
 * SALAD pages either.)
 */
int salad_check_status_static(salad_stream_t stream);

/*
 * The linear-branch state alone (summary section 2.1: ReLU linear attention),
 * computed by the same kernels salad_attn_forward uses:
 *   S_out  DEVICE fp32 [B*Hh][d][d], S[c][e] = sum_j relu(k_j[c]) v_j[e]
 *   z_out  DEVICE fp32 [B*Hh][d],    z[c]    = sum_j relu(k_j[c])
 *   gate   DEVICE fp32 [B][Hh] or NULL; (b, h) with gate 0 are skipped and their
 *          S/z rows are left untouched.
 * Same workspace rules as salad_attn_forward.  Errors as salad_attn_forward.
 */
int salad_linear_state(const void* k, const void* v, int B, int N, int num_heads, int d, const float* gate,
                       float* S_out, float* z_out, void* workspace, size_t workspace_bytes,
                       salad_stream_t stream);

/*
 * Synchronises `stream`, then reads and clears the workspace status word.
 * Returns SALAD_ERR_DEVICE_TIMEOUT if a kernel of an earlier call gave up on a
 * bounded wait (its output is then invalid), SALAD_ERR_BAD_MASK if a kernel of
 * the checking build (compiled with SALAD_DEBUG: libsalad_debug.so) found a
 * malformed mask row (a decreasing or out-of-range row_ptr, a column outside
 * [0, nb) or not ascending) and read it as an empty row, SALAD_ERR_CUDA if the
 * stream reports an error, SALAD_OK otherwise.  Release builds take mask rows
 * as given: check masks from elsewhere with salad_validate_mask first.
 */
int salad_check_status(void* workspace, salad_stream_t stream);

/*
 * Test hook: the longest time, in nanoseconds, a kernel waits on a pipeline
 * barrier before it records SALAD_ERR_DEVICE_TIMEOUT and returns.  The default
 * is 2 s; 0 makes every wait that is not already satisfied fail at once.
 * Affects launches made after the call (host-global setting).
 */
void salad_set_wait_limit_ns(uint64_t limit_ns);

/*
 * Test hook: the attention kernel is persistent (one CTA per SM, each taking
 * query tiles from a counter until none are left).  A positive value caps its
 * grid at max_ctas CTAs, so that small inputs also run many query tiles per
 * CTA; 0 restores one CTA per SM.  Host-global setting; it changes no result.
 */
void salad_set_max_ctas(int max_ctas);

/*
 * Profiling hook: caller-owned CUDA events (cudaEvent_t, passed as void*) that
 * subsequent salad_attn_forward calls record on their stream before the
 * linear-branch kernels, before the attention kernel and after it.  Pass NULLs
 * to stop.  Host-global setting; it changes no result.
 */
void salad_set_phase_events(void* before_linear, void* before_attention, void* after_attention);

/*
 * Profiling hook, live only in the profiling build of the library (compiled
 * with -DSALAD_PROFILE: `python -m sparse_linear_hybrid_b200.build --profile`,
 * which writes libsalad_profile.so); the normal build returns
 * SALAD_ERR_UNSUPPORTED and records nothing.  Later attention launches write
 * phase stamps (event code << 56 | SM clock) into `device_buffer`: per CTA,
 * 4 recording threads x 8192 uint64 words, for as many CTAs as `bytes` holds
 * (unused words keep what the caller put there).  NULL stops the recording.
 * sparse_linear_hybrid_b200/profile_phases.py reads them back as cycles per
 * phase.  Host-global setting; it changes no result.
 */
int salad_profile_set_buffer(void* device_buffer, size_t bytes);

const char* salad_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* SALAD_H_ */
