// C ABI of libsalad: argument validation, TMA tensor maps, launches, status.
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

using namespace salad;

namespace {

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_max_ctas{0};
std::atomic<void*> g_ev_linear{nullptr}, g_ev_attn{nullptr}, g_ev_end{nullptr};

bool record(const std::atomic<void*>& ev, cudaStream_t s) {
  void* e = ev.load();
  return e == nullptr || cudaEventRecord(static_cast<cudaEvent_t>(e), s) == cudaSuccess;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 tensor map, 128-byte swizzle, out-of-bounds elements read as zero.
bool make_map(CUtensorMap* m, const void* base, int rank, const uint64_t* dims, const uint64_t* strides_bytes,
              const uint32_t* box) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (rank < 1 || rank > 4) return false;
  cuuint64_t d[4];
  cuuint64_t st[3];
  cuuint32_t bx[4], es[4] = {1, 1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
  std::memset(m, 0, sizeof(*m));
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void*>(base), d, st, bx, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B][N][Hh][d] bf16 viewed as a 3-D tensor (Hh*d, N, B); box (64, rows, 1).
// With Hh_total > Hh the view is Hh consecutive heads of a tensor that holds
// Hh_total heads per token (`base` already points at the first of them).
bool make_bnhd_map(CUtensorMap* m, const void* base, int B, int N, int Hh, int d, uint32_t rows,
                   int Hh_total = 0) {
  const uint64_t row = (uint64_t)(Hh_total > 0 ? Hh_total : Hh) * d * 2;
  const uint64_t dims[3] = {(uint64_t)Hh * d, (uint64_t)N, (uint64_t)B};
  const uint64_t strides[2] = {row, (uint64_t)N * row};
  const uint32_t box[3] = {64, rows, 1};
  return make_map(m, base, 3, dims, strides, box);
}

// [B][T][H][W][Hh][d] bf16 viewed as a 4-D tensor (Hh*d, W, H, B*T); box
// (64, bw, bh, bt), one 3-D tile block of one head's 64-feature chunk.
bool make_tile_map(CUtensorMap* m, const void* base, int B, const TileGeom& g, int Hh, int d) {
  const uint64_t row = (uint64_t)Hh * d * 2;
  const uint64_t dims[4] = {(uint64_t)Hh * d, (uint64_t)g.W, (uint64_t)g.H, (uint64_t)B * g.T};
  const uint64_t strides[3] = {row, row * g.W, row * g.W * g.H};
  const uint32_t box[4] = {64, (uint32_t)g.bw, (uint32_t)g.bh, (uint32_t)g.bt};
  return make_map(m, base, 4, dims, strides, box);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Shared checks of salad_attn_forward / salad_linear_state.
int check_common(const void* k, const void* v, int B, int N, int Hh, int d, void* workspace,
                 size_t workspace_bytes) {
  if (!k || !v || !workspace) return SALAD_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || Hh < 1 || d < 1) return SALAD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SALAD_ERR_UNSUPPORTED;
  if (Hh > 65535 || (long long)B * Hh > 65535) return SALAD_ERR_UNSUPPORTED;
  if (!aligned(k, 16) || !aligned(v, 16) || !aligned(workspace, 256)) return SALAD_ERR_INVALID_ARG;
  if (workspace_bytes < workspace_layout(B, N, Hh, d).total) return SALAD_ERR_WORKSPACE;
  return SALAD_OK;
}

// The linear-branch kernels.  Forward (S_out == nullptr): z and (S W)^T into the
// workspace.  State export: S and z into S_out / z_out, with with_t also (S W)^T
// into the workspace.
int run_linear(const void* k, const void* v, int B, int N, int Hh, int d, const float* gate, const void* w_proj,
               float* S_out, float* z_out, uint8_t* ws, const WorkspaceLayout& L, cudaStream_t s, int Hh_total = 0,
               bool with_t = false) {
  CUtensorMap tk, tv;
  if (!make_bnhd_map(&tk, k, B, N, Hh, d, 64, Hh_total) || !make_bnhd_map(&tv, v, B, N, Hh, d, 64, Hh_total))
    return SALAD_ERR_CUDA;
  LinearArgs la{};
  la.tm_k = &tk;
  la.tm_v = &tv;
  la.gate = gate;
  la.partial = reinterpret_cast<float*>(ws + L.off_partial);
  la.w = static_cast<const uint16_t*>(w_proj);
  la.t_op = reinterpret_cast<uint16_t*>(ws + L.off_t);
  la.z = S_out ? z_out : reinterpret_cast<float*>(ws + L.off_z);
  la.S_out = S_out;
  la.with_t = with_t;
  la.work_ctr = reinterpret_cast<uint32_t*>(ws + L.off_status) + 1;
  la.B = B;
  la.N = N;
  la.heads = Hh;
  la.d = d;
  la.splits = L.splits;
  la.chunks_per_split = L.chunks_per_split;
  la.status = reinterpret_cast<uint32_t*>(ws + L.off_status);
  la.wait_limit_ns = g_wait_limit_ns.load();
  return launch_linear_reduce(la, s) == cudaSuccess ? SALAD_OK : SALAD_ERR_CUDA;
}

}  // namespace

extern "C" {

int salad_mask_num_blocks(int T, int H, int W, int block, int* nb) {
  if (!nb || T < 1 || H < 1 || W < 1 || block < 1) return SALAD_ERR_INVALID_ARG;
  const long long N = (long long)T * H * W;
  if (N >= (1ll << 31)) return SALAD_ERR_INVALID_ARG;
  *nb = (int)((N + block - 1) / block);
  return SALAD_OK;
}

namespace {
int build_mask_impl(int T, int H, int W, int block, int bt, int bh, int bw, int num_heads, const int32_t* windows,
                    int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int64_t* nnz_out,
                    salad_stream_t stream);
}

int salad_build_block_mask(int T, int H, int W, int block, int num_heads, const int32_t* windows,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int64_t* nnz_out,
                           salad_stream_t stream) {
  return build_mask_impl(T, H, W, block, 0, 0, 0, num_heads, windows, row_ptr, col_idx, col_capacity, nnz_out,
                         stream);
}

int salad_tile_num_blocks(int T, int H, int W, int bt, int bh, int bw, int* nb) {
  if (!nb || T < 1 || H < 1 || W < 1 || bt < 1 || bh < 1 || bw < 1) return SALAD_ERR_INVALID_ARG;
  if ((long long)T * H * W >= (1ll << 31)) return SALAD_ERR_INVALID_ARG;
  if (T % bt != 0) return SALAD_ERR_UNSUPPORTED;
  *nb = (T / bt) * ((H + bh - 1) / bh) * ((W + bw - 1) / bw);
  return SALAD_OK;
}

int salad_build_tile_mask(int T, int H, int W, int bt, int bh, int bw, int num_heads, const int32_t* windows,
                          int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int64_t* nnz_out,
                          salad_stream_t stream) {
  return build_mask_impl(T, H, W, 0, bt, bh, bw, num_heads, windows, row_ptr, col_idx, col_capacity, nnz_out,
                         stream);
}

}  // extern "C"

namespace {
int build_mask_impl(int T, int H, int W, int block, int bt, int bh, int bw, int num_heads, const int32_t* windows,
                    int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, int64_t* nnz_out,
                    salad_stream_t stream) {
  int nb = 0;
  int st = bt > 0 ? salad_tile_num_blocks(T, H, W, bt, bh, bw, &nb) : salad_mask_num_blocks(T, H, W, block, &nb);
  if (st != SALAD_OK) return st;
  if (!windows || !row_ptr || num_heads < 1 || num_heads > kMaxHeads || col_capacity < 0)
    return SALAD_ERR_INVALID_ARG;
  if (col_capacity > 0 && !col_idx) return SALAD_ERR_INVALID_ARG;
  if (!aligned(row_ptr, 4) || (col_idx && !aligned(col_idx, 4))) return SALAD_ERR_INVALID_ARG;
  // every kept pair must be addressable by an int32 offset
  if ((long long)num_heads * nb * nb >= (1ll << 31)) return SALAD_ERR_UNSUPPORTED;
  WindowTable win{};
  for (int h = 0; h < num_heads; ++h)
    for (int a = 0; a < 3; ++a) {
      if (windows[3 * h + a] < 0) return SALAD_ERR_INVALID_ARG;
      win.w[3 * h + a] = windows[3 * h + a];
    }
  MaskGrid g{T, H, W, bt > 0 ? bt * bh * bw : block, nb, num_heads, (long long)T * H * W};
  g.bt = bt;
  g.bh = bh;
  g.bw = bw;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (launch_mask_count(g, win, row_ptr, s) != cudaSuccess) return SALAD_ERR_CUDA;
  if (launch_mask_scan(row_ptr, num_heads * nb, s) != cudaSuccess) return SALAD_ERR_CUDA;
  int32_t total = 0;
  if (cudaMemcpyAsync(&total, row_ptr + (size_t)num_heads * nb, sizeof(total), cudaMemcpyDeviceToHost, s) !=
          cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SALAD_ERR_CUDA;
  if (nnz_out) *nnz_out = total;
  if (total > col_capacity) return SALAD_ERR_CAPACITY;
  if (total > 0 && launch_mask_fill(g, win, row_ptr, col_idx, s) != cudaSuccess) return SALAD_ERR_CUDA;
  return SALAD_OK;
}
}  // namespace

extern "C" {

size_t salad_workspace_bytes(int B, int N, int num_heads, int d) {
  if (B < 1 || N < 1 || num_heads < 1 || (d != 64 && d != 128)) return 0;
  return workspace_layout(B, N, num_heads, d).total;
}

}  // extern "C"

namespace {

int attn_forward_impl(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d, int block,
                      const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj, const float* gate,
                      float softmax_scale, float eps, void* out, void* workspace, size_t workspace_bytes,
                      salad_stream_t stream, int mask_per_bh, const TileGeom* tiles = nullptr,
                      float* lse = nullptr, int head_begin = 0, int heads_total = 0) {
  // heads_total > 0: q, k, v and out hold heads_total heads per token and the
  // call runs heads [head_begin, head_begin + num_heads) of them
  if (!q || !row_ptr || !col_idx || !w_proj || !gate || !out) return SALAD_ERR_INVALID_ARG;
  const int Ht = heads_total > 0 ? heads_total : num_heads;
  int st = check_common(k, v, B, N, num_heads, d, workspace, workspace_bytes);
  if (st != SALAD_OK) return st;
  if (block != 64 && block != 128) return SALAD_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(w_proj, 16) || !aligned(gate, 4) ||
      !aligned(row_ptr, 4) || !aligned(col_idx, 4))
    return SALAD_ERR_INVALID_ARG;
  if (!std::isfinite(eps) || eps < 0.f || !std::isfinite(softmax_scale)) return SALAD_ERR_INVALID_ARG;
  const size_t tensor_bytes = (size_t)B * N * Ht * d * 2;
  if (overlaps(out, tensor_bytes, q, tensor_bytes) || overlaps(out, tensor_bytes, k, tensor_bytes) ||
      overlaps(out, tensor_bytes, v, tensor_bytes))
    return SALAD_ERR_INVALID_ARG;
  // the first head of the range, as byte offsets into the tensors (16-byte
  // aligned: d is 64 or 128)
  const size_t h0 = (size_t)head_begin * d;
  q = static_cast<const uint16_t*>(q) + h0;
  k = static_cast<const uint16_t*>(k) + h0;
  v = static_cast<const uint16_t*>(v) + h0;
  out = static_cast<uint16_t*>(out) + h0;
  const long long qtiles = tiles ? (long long)(tiles->T / tiles->bt) * tiles->nh * tiles->nw : (N + 127) / 128;
  if (qtiles * B * num_heads >= (1ll << 31)) return SALAD_ERR_UNSUPPORTED;

  const WorkspaceLayout L = workspace_layout(B, N, num_heads, d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

  if (!record(g_ev_linear, s)) return SALAD_ERR_CUDA;
  st = run_linear(k, v, B, N, num_heads, d, gate, w_proj, nullptr, nullptr, ws, L, s, Ht);
  if (st != SALAD_OK) return st;

  CUtensorMap tq, tk, tv, to, tt;
  const int BH = B * num_heads;
  const uint64_t t_dims[3] = {(uint64_t)2 * d, (uint64_t)d, (uint64_t)BH};
  const uint64_t t_strides[2] = {(uint64_t)2 * d * 2, (uint64_t)d * 2 * d * 2};
  const uint32_t t_box[3] = {64, (uint32_t)d, 1};
  const bool maps_ok =
      tiles ? make_tile_map(&tq, q, B, *tiles, num_heads, d) && make_tile_map(&tk, k, B, *tiles, num_heads, d) &&
                  make_tile_map(&tv, v, B, *tiles, num_heads, d) && make_tile_map(&to, out, B, *tiles, num_heads, d)
            : make_bnhd_map(&tq, q, B, N, num_heads, d, 128, Ht) &&
                  make_bnhd_map(&tk, k, B, N, num_heads, d, block, Ht) &&
                  make_bnhd_map(&tv, v, B, N, num_heads, d, block, Ht) &&
                  make_bnhd_map(&to, out, B, N, num_heads, d, 128, Ht);
  if (!maps_ok || !make_map(&tt, ws + L.off_t, 3, t_dims, t_strides, t_box)) return SALAD_ERR_CUDA;

  AttnArgs aa{};
  aa.tm_q = &tq;
  aa.tm_k = &tk;
  aa.tm_v = &tv;
  aa.tm_out = &to;
  aa.tm_t = &tt;
  aa.row_ptr = row_ptr;
  aa.col_idx = col_idx;
  aa.gate = gate;
  aa.z = reinterpret_cast<const float*>(ws + L.off_z);
  aa.work_ctr = reinterpret_cast<uint32_t*>(ws + L.off_status) + 1;
  aa.max_ctas = g_max_ctas.load();
  aa.mask_per_bh = mask_per_bh;
  aa.tiles = tiles ? *tiles : TileGeom{};
  aa.lse = lse;
  aa.B = B;
  aa.N = N;
  aa.heads = num_heads;
  aa.d = d;
  aa.block = block;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)d);
  aa.scale_log2 = scale * 1.4426950408889634f;
  aa.eps = eps;
  aa.status = reinterpret_cast<uint32_t*>(ws + L.off_status);
  aa.wait_limit_ns = g_wait_limit_ns.load();
  if (!record(g_ev_attn, s)) return SALAD_ERR_CUDA;
  if (launch_attention(aa, s) != cudaSuccess) return SALAD_ERR_CUDA;
  return record(g_ev_end, s) ? SALAD_OK : SALAD_ERR_CUDA;
}

}  // namespace

extern "C" {

int salad_attn_forward(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d,
                       int block, const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj,
                       const float* gate, float softmax_scale, float eps, void* out, void* workspace,
                       size_t workspace_bytes, salad_stream_t stream) {
  return attn_forward_impl(q, k, v, B, N, num_heads, d, block, row_ptr, col_idx, w_proj, gate, softmax_scale, eps,
                           out, workspace, workspace_bytes, stream, 0);
}

int salad_attn_forward_bh(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d,
                          int block, const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj,
                          const float* gate, float softmax_scale, float eps, void* out, void* workspace,
                          size_t workspace_bytes, salad_stream_t stream) {
  return attn_forward_impl(q, k, v, B, N, num_heads, d, block, row_ptr, col_idx, w_proj, gate, softmax_scale, eps,
                           out, workspace, workspace_bytes, stream, 1);
}

int salad_attn_forward_lse(const void* q, const void* k, const void* v, int B, int N, int num_heads, int d,
                           int block, const int32_t* row_ptr, const int32_t* col_idx, const void* w_proj,
                           const float* gate, float softmax_scale, float eps, int mask_per_bh, void* out, float* lse,
                           void* workspace, size_t workspace_bytes, salad_stream_t stream) {
  if (!lse || !aligned(lse, 4)) return SALAD_ERR_INVALID_ARG;
  return attn_forward_impl(q, k, v, B, N, num_heads, d, block, row_ptr, col_idx, w_proj, gate, softmax_scale, eps,
                           out, workspace, workspace_bytes, stream, mask_per_bh ? 1 : 0, nullptr, lse);
}

int salad_attn_forward_heads(const void* q, const void* k, const void* v, int B, int N, int heads_total,
                             int head_begin, int head_count, int d, int block, const int32_t* row_ptr,
                             const int32_t* col_idx, const void* w_proj, const float* gate, float softmax_scale,
                             float eps, void* out, void* workspace, size_t workspace_bytes, salad_stream_t stream) {
  if (heads_total < 1 || head_begin < 0 || head_count < 1 || head_count > heads_total ||
      head_begin > heads_total - head_count)
    return SALAD_ERR_INVALID_ARG;
  if (heads_total > 65535) return SALAD_ERR_UNSUPPORTED;
  return attn_forward_impl(q, k, v, B, N, head_count, d, block, row_ptr, col_idx, w_proj, gate, softmax_scale, eps,
                           out, workspace, workspace_bytes, stream, 0, nullptr, nullptr, head_begin, heads_total);
}

int salad_attn_forward_host(const void* q_host, const void* k_host, const void* v_host, void* out_host, int B,
                            int N, int num_heads, int d, int block, const int32_t* row_ptr, const int32_t* col_idx,
                            const void* w_proj, const float* gate, float softmax_scale, float eps,
                            int heads_per_chunk, void* q_dev, void* k_dev, void* v_dev, void* out_dev,
                            void* workspace, size_t workspace_bytes, salad_stream_t stream,
                            salad_stream_t copy_in, salad_stream_t copy_out) {
  if (!q_host || !k_host || !v_host || !out_host || !q_dev || !k_dev || !v_dev || !out_dev || !row_ptr ||
      !col_idx || !w_proj || !gate || !workspace)
    return SALAD_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || num_heads < 1 || heads_per_chunk < 0) return SALAD_ERR_INVALID_ARG;
  if (block != 64 && block != 128) return SALAD_ERR_UNSUPPORTED;
  if (num_heads > 65535) return SALAD_ERR_UNSUPPORTED;
  // about six chunks per batch element: measured best at 12 heads (the last
  // chunk's compute and output copy are the part the copies cannot hide)
  int hpc = heads_per_chunk > 0 ? heads_per_chunk : (num_heads + 5) / 6;
  if (hpc > num_heads) hpc = num_heads;
  if (workspace_bytes < salad_workspace_bytes(1, N, hpc, d)) return SALAD_ERR_WORKSPACE;
  const void* p16[] = {q_dev, k_dev, v_dev, out_dev};
  for (const void* ptr : p16)
    if (!aligned(ptr, 16)) return SALAD_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaStream_t c_in = reinterpret_cast<cudaStream_t>(copy_in), c_out = reinterpret_cast<cudaStream_t>(copy_out);
  if (c_in == s || c_out == s || c_in == c_out) return SALAD_ERR_INVALID_ARG;
  const int nb = (N + block - 1) / block;
  const int chunks_per_b = (num_heads + hpc - 1) / hpc;
  const int chunks = B * chunks_per_b;
  // events ordering the three streams: the copies wait for the work queued on
  // `stream` before the call, each chunk's forward for its inputs, each chunk's
  // output copy for its forward, and `stream` for the last output copy
  std::vector<cudaEvent_t> ev(2 * (size_t)chunks + 2, nullptr);
  int st = SALAD_OK;
  for (auto& e : ev)
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      e = nullptr;
      st = SALAD_ERR_CUDA;
      break;
    }
  const size_t pitch = (size_t)num_heads * d * 2;
  auto bytes_at = [&](const void* base, size_t off) { return static_cast<const uint8_t*>(base) + off; };
  auto wbytes_at = [&](void* base, size_t off) { return static_cast<uint8_t*>(base) + off; };
  if (st == SALAD_OK &&
      (cudaEventRecord(ev[0], s) != cudaSuccess || cudaStreamWaitEvent(c_in, ev[0], 0) != cudaSuccess ||
       cudaStreamWaitEvent(c_out, ev[0], 0) != cudaSuccess))
    st = SALAD_ERR_CUDA;
  for (int c = 0; c < chunks && st == SALAD_OK; ++c) {
    const int b = c / chunks_per_b, h0 = (c % chunks_per_b) * hpc;
    const int hc = h0 + hpc <= num_heads ? hpc : num_heads - h0;
    const size_t batch_off = (size_t)b * N * pitch, off = batch_off + (size_t)h0 * d * 2;
    const size_t width = (size_t)hc * d * 2;
    const void* src[3] = {q_host, k_host, v_host};
    void* dst[3] = {q_dev, k_dev, v_dev};
    for (int t = 0; t < 3 && st == SALAD_OK; ++t)
      if (cudaMemcpy2DAsync(wbytes_at(dst[t], off), pitch, bytes_at(src[t], off), pitch, width, (size_t)N,
                            cudaMemcpyHostToDevice, c_in) != cudaSuccess)
        st = SALAD_ERR_CUDA;
    if (st != SALAD_OK) break;
    if (cudaEventRecord(ev[1 + 2 * c], c_in) != cudaSuccess || cudaStreamWaitEvent(s, ev[1 + 2 * c], 0) != cudaSuccess) {
      st = SALAD_ERR_CUDA;
      break;
    }
    // the chunk's forward: batch element b, heads [h0, h0 + hc) of the full tensors
    st = attn_forward_impl(bytes_at(q_dev, batch_off), bytes_at(k_dev, batch_off), bytes_at(v_dev, batch_off), 1, N,
                           hc, d, block, row_ptr + (size_t)h0 * nb, col_idx, w_proj, gate + (size_t)b * num_heads + h0,
                           softmax_scale, eps, wbytes_at(out_dev, batch_off), workspace, workspace_bytes, stream, 0,
                           nullptr, nullptr, h0, num_heads);
    if (st != SALAD_OK) break;
    if (cudaEventRecord(ev[2 + 2 * c], s) != cudaSuccess || cudaStreamWaitEvent(c_out, ev[2 + 2 * c], 0) != cudaSuccess ||
        cudaMemcpy2DAsync(wbytes_at(out_host, off), pitch, bytes_at(out_dev, off), pitch, width, (size_t)N,
                          cudaMemcpyDeviceToHost, c_out) != cudaSuccess)
      st = SALAD_ERR_CUDA;
  }
  // `stream` waits for the last output copy, so synchronising it covers the call
  if (st == SALAD_OK && (cudaEventRecord(ev.back(), c_out) != cudaSuccess ||
                         cudaStreamWaitEvent(s, ev.back(), 0) != cudaSuccess))
    st = SALAD_ERR_CUDA;
  for (auto e : ev)
    if (e != nullptr) cudaEventDestroy(e);  // released once the work recorded on it completes
  return st;
}

size_t salad_backward_workspace_bytes(int B, int N, int num_heads) {
  if (B < 1 || N < 1 || num_heads < 1) return 0;
  const size_t npad = ((size_t)N + 127) / 128 * 128;
  return 256 + 2 * (size_t)B * num_heads * npad * sizeof(float);
}

int salad_attn_backward_sparse(const void* q, const void* k, const void* v, const void* o, const void* dout,
                               const float* lse, int B, int N, int num_heads, int d, int block,
                               const int32_t* row_ptr, const int32_t* col_idx, const int32_t* t_row_ptr,
                               const int32_t* t_col_idx, int mask_per_bh, float softmax_scale, float* dq, float* dk,
                               float* dv, void* workspace, size_t workspace_bytes, salad_stream_t stream) {
  if (!q || !k || !v || !o || !dout || !lse || !row_ptr || !col_idx || !t_row_ptr || !t_col_idx || !dq || !dk ||
      !dv || !workspace)
    return SALAD_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || num_heads < 1) return SALAD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SALAD_ERR_UNSUPPORTED;
  if (block != 128) return SALAD_ERR_UNSUPPORTED;
  if (num_heads > 65535 || (long long)B * num_heads * ((N + 127) / 128) >= (1ll << 31)) return SALAD_ERR_UNSUPPORTED;
  const void* p16[] = {q, k, v, o, dout, dq, dk, dv, workspace};
  for (const void* ptr : p16)
    if (!aligned(ptr, 16)) return SALAD_ERR_INVALID_ARG;
  if (!aligned(lse, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(t_row_ptr, 4) ||
      !aligned(t_col_idx, 4))
    return SALAD_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale)) return SALAD_ERR_INVALID_ARG;
  if (workspace_bytes < salad_backward_workspace_bytes(B, N, num_heads)) return SALAD_ERR_WORKSPACE;
  CUtensorMap tq, tk, tv, tdo;
  if (!make_bnhd_map(&tq, q, B, N, num_heads, d, 128) || !make_bnhd_map(&tk, k, B, N, num_heads, d, 128) ||
      !make_bnhd_map(&tv, v, B, N, num_heads, d, 128) || !make_bnhd_map(&tdo, dout, B, N, num_heads, d, 128))
    return SALAD_ERR_CUDA;
  BwdArgs ba{};
  ba.tm_q = &tq;
  ba.tm_k = &tk;
  ba.tm_v = &tv;
  ba.tm_do = &tdo;
  ba.o = static_cast<const uint16_t*>(o);
  ba.dout = static_cast<const uint16_t*>(dout);
  ba.lse = lse;
  ba.row_ptr = row_ptr;
  ba.col_idx = col_idx;
  ba.t_row_ptr = t_row_ptr;
  ba.t_col_idx = t_col_idx;
  ba.B = B;
  ba.N = N;
  ba.heads = num_heads;
  ba.d = d;
  ba.nb = (N + 127) / 128;
  ba.npad = ba.nb * 128;
  ba.mask_per_bh = mask_per_bh ? 1 : 0;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  ba.status = reinterpret_cast<uint32_t*>(ws);
  ba.lse2 = reinterpret_cast<float*>(ws + 256);
  ba.dvec = ba.lse2 + (size_t)B * num_heads * ba.npad;
  ba.dq = dq;
  ba.dk = dk;
  ba.dv = dv;
  ba.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)d);
  ba.scale_log2 = ba.scale * 1.4426950408889634f;
  ba.wait_limit_ns = g_wait_limit_ns.load();
  return launch_backward(ba, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? SALAD_OK : SALAD_ERR_CUDA;
}

}  // extern "C"

namespace {
// Workspace of the layer backward (byte offsets; every region 256-byte aligned).
struct LayerBwdLayout {
  WorkspaceLayout fwd;  // the forward's workspace (status word at 0, (S W)^T, the state's partials)
  size_t off_S, off_z, off_lse2, off_dvec, off_mpart, off_dzpart, off_dgpart, off_dwpart, off_ds, off_dz, total;
  int splits, tiles_per_split, npad;
};
LayerBwdLayout layer_bwd_layout(int B, int N, int heads, int d) {
  LayerBwdLayout L{};
  L.fwd = workspace_layout(B, N, heads, d);
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t BH = (size_t)B * heads;
  L.npad = (N + 127) / 128 * 128;
  linear_backward_splits((int)BH, N, d, &L.splits, &L.tiles_per_split);
  const size_t S = (size_t)L.splits;
  size_t o = up(L.fwd.total);
  L.off_S = o;       o += up(BH * d * d * 4);
  L.off_z = o;       o += up(BH * d * 4);
  L.off_lse2 = o;    o += up(BH * L.npad * 4);
  L.off_dvec = o;    o += up(BH * L.npad * 4);
  L.off_mpart = o;   o += up(S * BH * d * d * 4);
  L.off_dzpart = o;  o += up(S * BH * 256 * 4);  // [splits][B*Hh][256/d row groups][d]
  L.off_dgpart = o;  o += up(S * BH * 4);
  L.off_dwpart = o;  o += up(BH * (d / 16) * d * d * 4);
  L.off_ds = o;      o += up(BH * d * 2 * d * 2);
  L.off_dz = o;      o += up(BH * d * 4);
  L.total = o;
  return L;
}
}  // namespace

extern "C" {

size_t salad_layer_backward_workspace_bytes(int B, int N, int num_heads, int d) {
  if (B < 1 || N < 1 || num_heads < 1 || (d != 64 && d != 128)) return 0;
  return layer_bwd_layout(B, N, num_heads, d).total;
}

int salad_attn_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                        const float* lse, int B, int N, int num_heads, int d, int block, const int32_t* row_ptr,
                        const int32_t* col_idx, const int32_t* t_row_ptr, const int32_t* t_col_idx, int mask_per_bh,
                        const void* w_proj, const float* gate, float softmax_scale, float eps, float* dq, float* dk,
                        float* dv, float* dw, float* dgate, void* workspace, size_t workspace_bytes,
                        salad_stream_t stream) {
  if (!q || !k || !v || !out || !dout || !lse || !row_ptr || !col_idx || !t_row_ptr || !t_col_idx || !w_proj ||
      !gate || !dq || !dk || !dv || !dw || !dgate || !workspace)
    return SALAD_ERR_INVALID_ARG;
  if (B < 1 || N < 1 || num_heads < 1) return SALAD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SALAD_ERR_UNSUPPORTED;
  if (block != 128) return SALAD_ERR_UNSUPPORTED;
  // (the streaming kernels run B*Hh rows of CTAs: at most 65535)
  if ((long long)B * num_heads > 65535 || (long long)B * num_heads * ((N + 127) / 128) >= (1ll << 31))
    return SALAD_ERR_UNSUPPORTED;
  const void* p16[] = {q, k, v, out, dout, w_proj, dq, dk, dv};
  for (const void* ptr : p16)
    if (!aligned(ptr, 16)) return SALAD_ERR_INVALID_ARG;
  if (!aligned(workspace, 256) || !aligned(lse, 4) || !aligned(gate, 4) || !aligned(dw, 4) || !aligned(dgate, 4) ||
      !aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(t_row_ptr, 4) || !aligned(t_col_idx, 4))
    return SALAD_ERR_INVALID_ARG;
  if (!std::isfinite(softmax_scale) || !std::isfinite(eps) || eps < 0.f) return SALAD_ERR_INVALID_ARG;
  const LayerBwdLayout L = layer_bwd_layout(B, N, num_heads, d);
  if (workspace_bytes < L.total) return SALAD_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  // 1. the linear branch's state S, z (fp32) and T = S W (bf16 hi + lo)
  int st = run_linear(k, v, B, N, num_heads, d, nullptr, w_proj, F(L.off_S), F(L.off_z), ws, L.fwd, s, 0, true);
  if (st != SALAD_OK) return st;
  CUtensorMap tq, tk, tv, tdo, tt, tds;
  const int BH = B * num_heads;
  const uint64_t op_dims[3] = {(uint64_t)2 * d, (uint64_t)d, (uint64_t)BH};
  const uint64_t op_strides[2] = {(uint64_t)2 * d * 2, (uint64_t)d * 2 * d * 2};
  const uint32_t op_box[3] = {64, (uint32_t)d, 1};
  if (!make_bnhd_map(&tq, q, B, N, num_heads, d, 128) || !make_bnhd_map(&tk, k, B, N, num_heads, d, 128) ||
      !make_bnhd_map(&tv, v, B, N, num_heads, d, 128) || !make_bnhd_map(&tdo, dout, B, N, num_heads, d, 128) ||
      !make_map(&tt, ws + L.fwd.off_t, 3, op_dims, op_strides, op_box) ||
      !make_map(&tds, ws + L.off_ds, 3, op_dims, op_strides, op_box))
    return SALAD_ERR_CUDA;
  LinBwdArgs la{};
  la.tm_q = &tq;
  la.tm_do = &tdo;
  la.tm_k = &tk;
  la.tm_v = &tv;
  la.tm_t = &tt;
  la.tm_ds = &tds;
  la.out = static_cast<const uint16_t*>(out);
  la.w = static_cast<const uint16_t*>(w_proj);
  la.lse = lse;
  la.gate = gate;
  la.S = F(L.off_S);
  la.z = F(L.off_z);
  la.dq = dq;
  la.dk = dk;
  la.dv = dv;
  la.dw = dw;
  la.dgate = dgate;
  la.lse2 = F(L.off_lse2);
  la.dvec = F(L.off_dvec);
  la.m_part = F(L.off_mpart);
  la.dz_part = F(L.off_dzpart);
  la.dg_part = F(L.off_dgpart);
  la.dw_part = F(L.off_dwpart);
  la.ds_op = reinterpret_cast<uint16_t*>(ws + L.off_ds);
  la.dz = F(L.off_dz);
  la.B = B;
  la.N = N;
  la.heads = num_heads;
  la.d = d;
  la.npad = L.npad;
  la.splits = L.splits;
  la.tiles_per_split = L.tiles_per_split;
  la.eps = eps;
  la.status = reinterpret_cast<uint32_t*>(ws + L.fwd.off_status);
  la.wait_limit_ns = g_wait_limit_ns.load();
  // 2. per-row terms of the linear branch, D_i and lse2; dq starts as the linear branch's part
  if (launch_linear_backward_rows(la, s) != cudaSuccess) return SALAD_ERR_CUDA;
  // 3. dS, dz, dW, dgate
  if (launch_linear_backward_state(la, s) != cudaSuccess) return SALAD_ERR_CUDA;
  // 4. the sparse branch: dq += ..., dk and dv written
  BwdArgs ba{};
  ba.tm_q = &tq;
  ba.tm_k = &tk;
  ba.tm_v = &tv;
  ba.tm_do = &tdo;
  ba.o = static_cast<const uint16_t*>(out);
  ba.dout = static_cast<const uint16_t*>(dout);
  ba.lse = lse;
  ba.row_ptr = row_ptr;
  ba.col_idx = col_idx;
  ba.t_row_ptr = t_row_ptr;
  ba.t_col_idx = t_col_idx;
  ba.lse2 = la.lse2;
  ba.dvec = la.dvec;
  ba.dq = dq;
  ba.dk = dk;
  ba.dv = dv;
  ba.B = B;
  ba.N = N;
  ba.heads = num_heads;
  ba.d = d;
  ba.nb = L.npad / 128;
  ba.npad = L.npad;
  ba.mask_per_bh = mask_per_bh ? 1 : 0;
  ba.scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)d);
  ba.scale_log2 = ba.scale * 1.4426950408889634f;
  ba.status = reinterpret_cast<uint32_t*>(ws + L.fwd.off_status);
  ba.wait_limit_ns = g_wait_limit_ns.load();
  ba.full = 1;
  if (launch_backward(ba, s) != cudaSuccess) return SALAD_ERR_CUDA;
  // 5. the linear parts of dk and dv
  return launch_linear_backward_keys(la, s) == cudaSuccess ? SALAD_OK : SALAD_ERR_CUDA;
}

int salad_attn_forward_tiles(const void* q, const void* k, const void* v, int B, int T, int H, int W, int bt,
                             int bh, int bw, int num_heads, int d, const int32_t* row_ptr, const int32_t* col_idx,
                             const void* w_proj, const float* gate, float softmax_scale, float eps, void* out,
                             void* workspace, size_t workspace_bytes, salad_stream_t stream) {
  int nb = 0;
  const int st = salad_tile_num_blocks(T, H, W, bt, bh, bw, &nb);
  if (st != SALAD_OK) return st;
  if (bt * bh * bw != 128) return SALAD_ERR_UNSUPPORTED;
  TileGeom g{T, H, W, bt, bh, bw, (H + bh - 1) / bh, (W + bw - 1) / bw, {}, {}};
  // the kernel divides box indices (< nb) by nw and row indices (< nb / nw) by
  // nh with multiply-high divisors, exact while n * divisor < 2^32
  if ((uint64_t)nb * g.nw >= (1ull << 32) || (uint64_t)nb * g.nh >= (1ull << 32)) return SALAD_ERR_UNSUPPORTED;
  g.div_nw = make_fastdiv((uint32_t)g.nw);
  g.div_nh = make_fastdiv((uint32_t)g.nh);
  return attn_forward_impl(q, k, v, B, T * H * W, num_heads, d, 128, row_ptr, col_idx, w_proj, gate, softmax_scale,
                           eps, out, workspace, workspace_bytes, stream, 0, &g);
}

int salad_transpose_block_mask(const int32_t* row_ptr, const int32_t* col_idx, int groups, int nb,
                               int32_t* t_row_ptr, int32_t* t_col_idx, salad_stream_t stream) {
  if (!row_ptr || !col_idx || !t_row_ptr || !t_col_idx || groups < 1 || nb < 1) return SALAD_ERR_INVALID_ARG;
  if (!aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(t_row_ptr, 4) || !aligned(t_col_idx, 4))
    return SALAD_ERR_INVALID_ARG;
  // (one CTA row per group; every pair must be addressable by an int32 offset)
  if (groups > 65535 || (long long)groups * nb * nb >= (1ll << 31)) return SALAD_ERR_UNSUPPORTED;
  return launch_mask_transpose(row_ptr, col_idx, groups, nb, t_row_ptr, t_col_idx, nullptr,
                               reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SALAD_OK
             : SALAD_ERR_CUDA;
}

int salad_validate_mask(const int32_t* row_ptr, const int32_t* col_idx, int64_t rows, int nb, int64_t* bad_row) {
  if (bad_row) *bad_row = -1;
  if (!row_ptr || rows < 0 || nb < 1) return SALAD_ERR_INVALID_ARG;
  if (row_ptr[0] != 0) {
    if (bad_row) *bad_row = 0;
    return SALAD_ERR_INVALID_ARG;
  }
  for (int64_t r = 0; r < rows; ++r) {
    const int32_t a = row_ptr[r], e = row_ptr[r + 1];
    bool ok = e >= a && e - a <= nb && (e == a || col_idx != nullptr);
    for (int32_t i = a; ok && i < e; ++i)
      ok = col_idx[i] >= 0 && col_idx[i] < nb && (i == a || col_idx[i] > col_idx[i - 1]);
    if (!ok) {
      if (bad_row) *bad_row = r;
      return SALAD_ERR_INVALID_ARG;
    }
  }
  return SALAD_OK;
}

size_t salad_gate_workspace_bytes(int B, int N, int num_heads, int d) {
  if (B < 1 || N < 1 || num_heads < 1 || (d != 64 && d != 128)) return 0;
  return gate_workspace_bytes(B, N, num_heads, d);
}

int salad_gate_forward(const void* q, int B, int N, int num_heads, int d, const float* t_emb, int E,
                       const float* w_t, const float* w_x, const float* beta, float threshold, float* s_out,
                       float* gate_out, void* workspace, size_t workspace_bytes, salad_stream_t stream) {
  if (!q || !w_x || !beta || !gate_out || !workspace || B < 1 || N < 1 || num_heads < 1 || E < 0)
    return SALAD_ERR_INVALID_ARG;
  if (E > 0 && (!t_emb || !w_t)) return SALAD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SALAD_ERR_UNSUPPORTED;
  if (B > 65535 || (long long)B * num_heads >= (1ll << 31)) return SALAD_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(workspace, 16) || !aligned(gate_out, 4) || (s_out && !aligned(s_out, 4)))
    return SALAD_ERR_INVALID_ARG;
  if (!std::isfinite(threshold)) return SALAD_ERR_INVALID_ARG;
  if (workspace_bytes < gate_workspace_bytes(B, N, num_heads, d)) return SALAD_ERR_WORKSPACE;
  GateArgs ga{};
  ga.q = static_cast<const uint16_t*>(q);
  ga.B = B;
  ga.N = N;
  ga.heads = num_heads;
  ga.d = d;
  ga.E = E;
  ga.t_emb = t_emb;
  ga.w_t = w_t;
  ga.w_x = w_x;
  ga.beta = beta;
  ga.threshold = threshold;
  ga.partial = static_cast<float*>(workspace);
  ga.s_out = s_out;
  ga.gate_out = gate_out;
  return launch_gate(ga, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? SALAD_OK : SALAD_ERR_CUDA;
}

size_t salad_topk_workspace_bytes(int B, int N, int num_heads, int d, int block) {
  if (B < 1 || N < 1 || num_heads < 1 || (d != 64 && d != 128) || block < 1) return 0;
  return topk_workspace_bytes(B, N, num_heads, d, block);
}

int salad_build_topk_mask(const void* q, const void* k, int B, int N, int num_heads, int d, int block, int keep,
                          int32_t* row_ptr, int32_t* col_idx, void* workspace, size_t workspace_bytes,
                          salad_stream_t stream) {
  if (!q || !k || !row_ptr || !col_idx || !workspace || B < 1 || N < 1 || num_heads < 1 || block < 1 || keep < 1)
    return SALAD_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SALAD_ERR_UNSUPPORTED;
  const long long nb = ((long long)N + block - 1) / block;
  if (nb > kTopkMaxBlocks) return SALAD_ERR_UNSUPPORTED;
  const long long kk = keep < nb ? keep : nb;
  // (the pooling launches B*Hh rows of CTAs: at most 65535)
  if ((long long)B * num_heads > 65535 || (long long)B * num_heads * nb * kk >= (1ll << 31) ||
      (long long)B * N * num_heads * d >= (1ll << 40))
    return SALAD_ERR_UNSUPPORTED;
  if (!aligned(q, 4) || !aligned(k, 4) || !aligned(row_ptr, 4) || !aligned(col_idx, 4) || !aligned(workspace, 4))
    return SALAD_ERR_INVALID_ARG;
  if (workspace_bytes < topk_workspace_bytes(B, N, num_heads, d, block)) return SALAD_ERR_WORKSPACE;
  TopkArgs ta{};
  ta.q = static_cast<const uint16_t*>(q);
  ta.k = static_cast<const uint16_t*>(k);
  ta.B = B;
  ta.N = N;
  ta.heads = num_heads;
  ta.d = d;
  ta.block = block;
  ta.nb = (int)nb;
  ta.kk = (int)kk;
  ta.qm = static_cast<float*>(workspace);
  ta.km = ta.qm + (size_t)B * num_heads * nb * d;
  ta.row_ptr = row_ptr;
  ta.col_idx = col_idx;
  return launch_topk_mask(ta, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? SALAD_OK : SALAD_ERR_CUDA;
}

int salad_linear_state(const void* k, const void* v, int B, int N, int num_heads, int d, const float* gate,
                       float* S_out, float* z_out, void* workspace, size_t workspace_bytes,
                       salad_stream_t stream) {
  if (!S_out || !z_out) return SALAD_ERR_INVALID_ARG;
  int st = check_common(k, v, B, N, num_heads, d, workspace, workspace_bytes);
  if (st != SALAD_OK) return st;
  if ((gate && !aligned(gate, 4)) || !aligned(S_out, 4) || !aligned(z_out, 4)) return SALAD_ERR_INVALID_ARG;
  const WorkspaceLayout L = workspace_layout(B, N, num_heads, d);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  return run_linear(k, v, B, N, num_heads, d, gate, nullptr, S_out, z_out, ws, L, s);
}

int salad_check_status(void* workspace, salad_stream_t stream) {
  if (!workspace) return SALAD_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SALAD_ERR_CUDA;
  uint32_t word = 0;
  uint32_t* dev = static_cast<uint32_t*>(workspace);
  if (cudaMemcpyAsync(&word, dev, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return SALAD_ERR_CUDA;
  if (word == 0) return SALAD_OK;
  if (cudaMemsetAsync(dev, 0, sizeof(word), s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
    return SALAD_ERR_CUDA;
  if (word & kStatusTimeout) return SALAD_ERR_DEVICE_TIMEOUT;
  return (word & kStatusBadMask) ? SALAD_ERR_BAD_MASK : SALAD_ERR_CUDA;
}

void salad_set_wait_limit_ns(uint64_t limit_ns) { g_wait_limit_ns.store(limit_ns); }

void salad_set_max_ctas(int max_ctas) { g_max_ctas.store(max_ctas > 0 ? max_ctas : 0); }

int salad_profile_set_buffer(void* device_buffer, size_t bytes) {
  if (device_buffer != nullptr && (reinterpret_cast<uintptr_t>(device_buffer) % 8) != 0)
    return SALAD_ERR_INVALID_ARG;
  return set_profile_buffer(device_buffer, device_buffer ? bytes : 0);
}

void salad_set_phase_events(void* before_linear, void* before_attention, void* after_attention) {
  g_ev_linear.store(before_linear);
  g_ev_attn.store(before_attention);
  g_ev_end.store(after_attention);
}

const char* salad_status_string(int status) {
  switch (status) {
    case SALAD_OK: return "ok";
    case SALAD_ERR_INVALID_ARG: return "invalid argument";
    case SALAD_ERR_UNSUPPORTED: return "unsupported configuration";
    case SALAD_ERR_CAPACITY: return "col_idx capacity too small";
    case SALAD_ERR_WORKSPACE: return "workspace too small";
    case SALAD_ERR_CUDA: return "CUDA error";
    case SALAD_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case SALAD_ERR_BAD_MASK: return "a kernel skipped a malformed mask row (checking build)";
    case SALAD_ERR_OUT_OF_MEMORY: return "device out of memory for the static scratch";
    default: return "unknown status";
  }
}

}  // extern "C"
