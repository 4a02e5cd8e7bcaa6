// salad_attn_forward_static: the layer forward with its workspace in a static
// device array instead of caller-provided memory.
//
// Some callers cannot call cudaMalloc: a plugin running inside a serving engine
// that reserves the whole device memory pool up front and forbids further
// allocations, or a latency-critical path that may not pay cudaMalloc's
// implicit device synchronisation.  This entry point lets them run the layer
// with nothing but their inputs and outputs: the scratch the forward needs (the
// status word, the linear-branch state [S | z] and the split partial sums)
// lives in the file-scope array below, which every GPU that loads the library
// holds until the process exits.
#include <mutex>

#include "internal.h"

namespace {

static __device__ __align__(256) uint8_t g_static_scratch[SALAD_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the static scratch on the current device.  Host code only
// sees a host-side stand-in under the array's name, so the address is looked
// up once per device, with that device current, and cached.
int scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SALAD_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return SALAD_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SALAD_OK;
}

}  // namespace

extern "C" int salad_attn_forward_static(const void* q, const void* k, const void* v, int B, int N, int num_heads,
                                         int d, int block, const int32_t* row_ptr, const int32_t* col_idx,
                                         const void* w_proj, const float* gate, float softmax_scale, float eps,
                                         void* out, salad_stream_t stream) {
  const size_t need = salad_workspace_bytes(B, N, num_heads, d);
  if (need == 0) return (B < 1 || N < 1 || num_heads < 1 || d < 1) ? SALAD_ERR_INVALID_ARG : SALAD_ERR_UNSUPPORTED;
  if (need > SALAD_STATIC_SCRATCH_BYTES) return SALAD_ERR_WORKSPACE;
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != SALAD_OK) return st;
  // the array keeps the previous call's contents; only the status word must
  // start at zero (every other byte the forward reads it first writes)
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t), s) != cudaSuccess) return SALAD_ERR_CUDA;
  return salad_attn_forward(q, k, v, B, N, num_heads, d, block, row_ptr, col_idx, w_proj, gate, softmax_scale,
                            eps, out, scratch, SALAD_STATIC_SCRATCH_BYTES, stream);
}
