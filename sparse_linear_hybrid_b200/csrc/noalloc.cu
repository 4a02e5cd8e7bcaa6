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
#include "internal.h"

namespace {

// Zero-initialised when the module is loaded on a device, so its status word
// starts at 0; afterwards only salad_check_status_static clears it.
static __device__ __align__(256) uint8_t g_static_scratch[SALAD_STATIC_SCRATCH_BYTES];

// Device address of the static scratch on the current device.  Host code only
// sees a host-side stand-in under the array's name, so the address is asked of
// the runtime with the device current.  It is asked on every call rather than
// cached: a context that is reset and created again loads the module anew, at
// an address a cached value would not follow.  The first lookup on a device
// loads the module, which maps the array's memory; the runtime reports a
// failure to map it as an allocation error.
int scratch_address(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
  if (e == cudaErrorMemoryAllocation) {
    (void)cudaGetLastError();  // not sticky: clear it so the caller's next call is unaffected
    return SALAD_ERR_OUT_OF_MEMORY;
  }
  if (e != cudaSuccess || p == nullptr) return SALAD_ERR_CUDA;
  *out = p;
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
  // The array keeps the previous call's contents.  Every byte the forward reads
  // it first writes, except the status word, which records a time-out until
  // salad_check_status_static reads and clears it (as the workspace forward's
  // does until salad_check_status).
  return salad_attn_forward(q, k, v, B, N, num_heads, d, block, row_ptr, col_idx, w_proj, gate, softmax_scale,
                            eps, out, scratch, SALAD_STATIC_SCRATCH_BYTES, stream);
}

extern "C" int salad_check_status_static(salad_stream_t stream) {
  void* scratch = nullptr;
  const int st = scratch_address(&scratch);
  if (st != SALAD_OK) return st;
  return salad_check_status(scratch, stream);
}
