// Internal declarations shared by the libsalad translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstddef>
#include <cstdint>

#include "../../include/salad.h"

namespace salad {

constexpr int kMaxHeads = 256;

// Window table passed by value to the mask kernels (kMaxHeads * 12 bytes).
struct WindowTable {
  int32_t w[3 * kMaxHeads];
};

struct MaskGrid {
  int T, H, W, block, nb, heads;
  long long N;
  int bt = 0, bh = 0, bw = 0;  // 3-D tile blocks of bt x bh x bw points (bt = 0: raster blocks of `block` tokens)
};

cudaError_t launch_mask_count(const MaskGrid& g, const WindowTable& win, int32_t* row_ptr, cudaStream_t s);
cudaError_t launch_mask_scan(int32_t* row_ptr, int n, cudaStream_t s);
cudaError_t launch_mask_fill(const MaskGrid& g, const WindowTable& win, const int32_t* row_ptr, int32_t* col_idx,
                             cudaStream_t s);
// The transposed mask of `groups` x nb rows (count, scan, fill).
// status: a device word for debug builds' kStatusBadMask bit, or null.
cudaError_t launch_mask_transpose(const int32_t* row_ptr, const int32_t* col_idx, int groups, int nb,
                                  int32_t* t_row_ptr, int32_t* t_col_idx, uint32_t* status, cudaStream_t s);

// Workspace layout of the forward pass (byte offsets from the workspace base).
struct WorkspaceLayout {
  int splits;             // split-N factor of the linear-branch reduction
  int chunks_per_split;   // 64-token chunks per split
  size_t off_status;      // uint32 status word, then the uint32 work counter of the attention kernel
  size_t off_t;           // bf16 [B*Hh][d][2d]: (S W)^T split into hi and lo halves
  size_t off_z;           // fp32 [B*Hh][d]: z
  size_t off_partial;     // fp32 [splits][B*Hh][d+1][d]: per-split S rows, then z
  size_t total;
};
WorkspaceLayout workspace_layout(int B, int N, int heads, int d);

struct LinearArgs {
  const CUtensorMap* tm_k;  // box (64, 64 tokens, 1)
  const CUtensorMap* tm_v;
  const float* gate;        // nullable
  float* partial;
  const uint16_t* w;        // forward: bf16 [d][d] projection
  uint16_t* t_op;           // forward: (S W)^T hi | lo, bf16 [B*Hh][d][2d]
  float* z;                 // fp32 [B*Hh][d]
  float* S_out;             // state export: fp32 [B*Hh][d][d]; null in the forward
  bool with_t = false;      // with S_out: also (S W)^T into t_op (the layer backward)
  uint32_t* work_ctr;       // zeroed here for the attention kernel that follows
  int B, N, heads, d, splits, chunks_per_split;
  uint32_t* status;
  uint64_t wait_limit_ns;
};
cudaError_t launch_linear_reduce(const LinearArgs& a, cudaStream_t s);

// 3-D tile blocks: box I = (ti*nh + yi)*nw + xi holds the points
// [ti*bt, +bt) x [yi*bh, +bh) x [xi*bw, +bw) of the T x H x W grid, slot
// (tt*bh + yy)*bw + xx.  bt == 0: raster blocks of consecutive tokens.
// Division by a fixed d >= 1 without the divide sequence: for n * d < 2^32,
// n / d == umulhi(n, m) with m = floor(2^32 / d) + 1 (d >= 2; the error term
// n * (m - 2^32 / d) / 2^32 stays below 1 / d), and n itself when d == 1
// (m = 0, one = all ones).
struct FastDiv {
  uint32_t m, one;
};
inline FastDiv make_fastdiv(uint32_t d) {
  return d <= 1 ? FastDiv{0u, 0xFFFFFFFFu} : FastDiv{(uint32_t)((1ull << 32) / d + 1), 0u};
}
#ifdef __CUDACC__
__device__ __forceinline__ uint32_t fastdiv(uint32_t n, FastDiv f) { return __umulhi(n, f.m) + (n & f.one); }
#endif

struct TileGeom {
  int T, H, W, bt, bh, bw, nh, nw;
  FastDiv div_nw, div_nh;  // box index -> (t*nh + y, x) -> (t, y)
};

struct AttnArgs {
  const CUtensorMap* tm_q;    // box (64, 128, 1); with tile blocks (Hh*d, W, H, B*T), box (64, bw, bh, bt)
  const CUtensorMap* tm_k;    // box (64, block, 1)
  const CUtensorMap* tm_v;    // box (64, block, 1)
  const CUtensorMap* tm_out;  // box (64, 128, 1)
  const CUtensorMap* tm_t;    // box (64, d, 1) over (S W)^T hi | lo
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const float* gate;
  const float* z;             // fp32 [B*Hh][d]
  uint32_t* work_ctr;         // next work item (zeroed by the linear kernel)
  int max_ctas;               // cap on the persistent grid (0: one CTA per SM)
  int mask_per_bh;            // mask rows are (b*Hh + h, I) instead of (h, I)
  TileGeom tiles;             // tiles.bt > 0: blocks are 3-D boxes (block == 128), maps are 4-D
  float* lse;                 // fp32 [B*Hh][N]: each row's log-sum-exp of the sparse softmax, or nullptr
  int B, N, heads, d, block;
  float scale_log2;  // softmax scale * log2(e)
  float eps;
  uint32_t* status;
  uint64_t wait_limit_ns;
};
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s);
// Profiling build only (SALAD_PROFILE): the attention kernel's phase-stamp
// buffer; SALAD_ERR_UNSUPPORTED in the normal build.
int set_profile_buffer(void* dev, size_t bytes);

// Backward pass of the sparse branch (bwd.cu); raster blocks of 128 tokens.
struct BwdArgs {
  const CUtensorMap *tm_q, *tm_k, *tm_v, *tm_do;  // box (64, 128, 1)
  const uint16_t* o;     // bf16 [B][N][Hh][d]: the branch output
  const uint16_t* dout;  // bf16 [B][N][Hh][d]
  const float* lse;      // fp32 [B*Hh][N], natural log
  const int32_t *row_ptr, *col_idx;      // mask rows (query block -> kept key blocks)
  const int32_t *t_row_ptr, *t_col_idx;  // its transpose (key block -> query blocks that keep it)
  float *lse2, *dvec;    // workspace: fp32 [B*Hh][npad] each
  float *dq, *dk, *dv;   // fp32 [B][N][Hh][d]
  int B, N, heads, d, nb, npad, mask_per_bh;
  float scale, scale_log2;
  uint32_t* status;
  uint64_t wait_limit_ns;
  int full = 0;  // with the linear branch: D_i and lse2 come from the row kernel, dq is added to
};
cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s);

// Backward pass of the linear branch, projection and gate (bwd_linear.cu).
struct LinBwdArgs {
  const CUtensorMap *tm_q, *tm_do, *tm_k, *tm_v;  // box (64, 128, 1)
  const CUtensorMap* tm_t;                         // box (64, d, 1) over (S W)^T hi | lo (the forward's layout)
  const CUtensorMap* tm_ds;                        // box (64, d, 1) over ds_op
  const uint16_t *out, *w;                         // bf16
  const float *lse, *gate, *S, *z;                 // S fp32 [B*Hh][d][d], z [B*Hh][d]
  float *dq, *dk, *dv, *dw, *dgate;
  float *lse2, *dvec;                              // [B*Hh][npad], read by the sparse backward
  float *m_part, *dz_part, *dg_part;               // [splits][B*Hh][d][d], [splits][B*Hh][256/d][d], [splits][B*Hh]
  float* dw_part;                                  // [B*Hh][d/16][d][d]
  uint16_t* ds_op;                                 // bf16 [B*Hh][d][2d]: dS hi | lo, rows c
  float* dz;                                       // [B*Hh][d]
  int B, N, heads, d, npad, splits, tiles_per_split;
  float eps;
  uint32_t* status;
  uint64_t wait_limit_ns;
};
// Splits of the streaming kernels: CTAs per (b, h) and 128-row tiles per CTA.
void linear_backward_splits(int BH, int N, int d, int* splits, int* tiles_per_split);
// dq (linear part), D_i, lse2 and the per-split M, dz, dgate.
cudaError_t launch_linear_backward_rows(const LinBwdArgs& a, cudaStream_t s);
// dS operand, dz, dgate, dW.
cudaError_t launch_linear_backward_state(const LinBwdArgs& a, cudaStream_t s);
// dk, dv += the linear parts.
cudaError_t launch_linear_backward_keys(const LinBwdArgs& a, cudaStream_t s);

// Dynamic gate and branch dropping (gate.cu).
struct GateArgs {
  const uint16_t* q;  // bf16 [B][N][Hh][d], 16-byte aligned
  int B, N, heads, d, E;
  const float* t_emb;  // [B][E]
  const float* w_t;    // [Hh][E]
  const float* w_x;    // [Hh][d]
  const float* beta;   // [Hh]
  float threshold;
  float* partial;      // workspace: [splits][B][Hh*d]
  float* s_out;        // [B][Hh] or nullptr
  float* gate_out;     // [B][Hh]
};
int gate_splits(int B, int N, int* chunk);
size_t gate_workspace_bytes(int B, int N, int heads, int d);
cudaError_t launch_gate(const GateArgs& a, cudaStream_t s);

// Top-K dynamic block mask (topk.cu).
struct TopkArgs {
  const uint16_t* q;  // bf16 [B][N][Hh][d]
  const uint16_t* k;
  int B, N, heads, d, block, nb, kk;  // kk = min(keep, nb) blocks kept per row
  float* qm;                          // fp32 [B*Hh][nb][d] block means of q (workspace)
  float* km;                          // and of k
  int32_t* row_ptr;                   // [B*Hh*nb + 1]
  int32_t* col_idx;                   // [B*Hh*nb*kk]
};
size_t topk_workspace_bytes(int B, int N, int heads, int d, int block);
cudaError_t launch_topk_mask(const TopkArgs& a, cudaStream_t s);
constexpr int kTopkMaxBlocks = 2048;  // the selection keeps one row of scores per query block in shared memory

// Status word bits written by kernels.
constexpr uint32_t kStatusTimeout = 1u;
constexpr uint32_t kStatusBadMask = 2u;  // debug builds: a malformed mask row was skipped

#ifdef __CUDACC__
// Debug builds (SALAD_DEBUG) check a CSR row of a block mask before a kernel
// indexes with it: 0 <= row_ptr[r] <= row_ptr[r + 1] <= row_ptr[rows] and, with
// cols, every column in [0, nb) and strictly ascending.  A bad row sets
// kStatusBadMask (where the call has a status word) and the caller treats it as
// empty, so no access follows from it; the kernel goes on with the other rows.  Release builds take every row
// as given (the host validates masks with salad_validate_mask).
__device__ __forceinline__ bool debug_row_ok(const int32_t* row_ptr, const int32_t* col_idx, int r, int rows,
                                             int nb, bool cols, uint32_t* status) {
#ifdef SALAD_DEBUG
  const int32_t lo = row_ptr[r], hi = row_ptr[r + 1], total = row_ptr[rows];
  bool ok = r >= 0 && r < rows && 0 <= lo && lo <= hi && hi <= total;
  for (int32_t i = lo; cols && ok && i < hi; ++i) {
    const int32_t c = col_idx[i];
    ok = c >= 0 && c < nb && (i == lo || c > col_idx[i - 1]);
  }
  if (!ok && status != nullptr) atomicOr(status, kStatusBadMask);
  return ok;
#else
  (void)row_ptr, (void)col_idx, (void)r, (void)rows, (void)nb, (void)cols, (void)status;
  return true;
#endif
}
#endif

}  // namespace salad
