// The dynamic gate of the linear branch and branch dropping (SALAD technical
// summary, section 2.2 ITADS: a lightweight module turns the denoising
// timestep and the hidden state into a global factor through a sigmoid;
// section 2.3: at inference the branch is dropped where that factor is very
// low).  The module implemented (include/salad.h states it): per (b, h)
//   s = sigmoid(w_t[h] . t_emb[b] + w_x[h] . mean_n q[b][n][h][:] + beta[h]),
//   gate = 0 where s < threshold (the linear branch is then skipped), else s.
//
// gate_pool_kernel      grid (splits, B), 192 x 4 threads: each CTA sums q over
//                       its run of tokens for every (h, feature) into fp32
//                       partials [splits][B][Hh*d]: four interleaved token
//                       streams (thread row r takes tokens r, r + 4, ...), each
//                       in token order, added in stream order (16-byte loads of
//                       the [Hh*d] token row, coalesced across threads).
// gate_finalize_kernel  grid (B*Hh), 1024 threads: eight groups of 128 threads
//                       each sum every eighth split's partials in split order,
//                       the groups are added in order; then the mean, the two
//                       dot products as fixed-order tree sums, the sigmoid and
//                       the threshold.
// Memory: q is read once (2*Hh*d bytes per token); the rest is small.
#include "internal.h"

namespace salad {
namespace {

constexpr int kPoolThreads = 192;  // 16-byte column chunks of a token row side by side
constexpr int kPoolRows = 4;       // interleaved token streams
constexpr int kFinThreads = 128;  // the features' share of the finalize CTA (d <= 128)
constexpr int kFinGroups = 8;     // split groups summed side by side

__global__ void __launch_bounds__(kPoolThreads* kPoolRows) gate_pool_kernel(const uint4* __restrict__ q, int N,
                                                                            int C8, int chunk,
                                                                            float* __restrict__ partial) {
  __shared__ float rows[kPoolRows - 1][kPoolThreads][8];
  const int split = blockIdx.x, b = blockIdx.y, r = threadIdx.y;
  const int n0 = split * chunk, n1 = min(N, n0 + chunk);
  float* dst = partial + ((size_t)split * gridDim.y + b) * (size_t)C8 * 8;
  for (int c0 = 0; c0 < C8; c0 += kPoolThreads) {
    const int c = c0 + threadIdx.x;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (c < C8) {
      const uint4* src = q + ((size_t)b * N + n0 + r) * C8 + c;
#pragma unroll 8
      for (int n = n0 + r; n < n1; n += kPoolRows, src += (size_t)kPoolRows * C8) {
        const uint4 x = *src;
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] += __uint_as_float(w[i] << 16);
          acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
    }
    if (r > 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) rows[r - 1][threadIdx.x][i] = acc[i];
    }
    __syncthreads();
    if (r == 0 && c < C8) {
#pragma unroll
      for (int k = 0; k < kPoolRows - 1; ++k)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] += rows[k][threadIdx.x][i];
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[(size_t)c * 8 + i] = acc[i];
    }
    __syncthreads();
  }
}

// Fixed-order tree sum of the values of the first kFinThreads threads (every
// thread of the block calls it).
__device__ float block_sum(float v, float* red) {
  if (threadIdx.x < kFinThreads) red[threadIdx.x] = v;
  __syncthreads();
#pragma unroll
  for (int s = kFinThreads / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const float r = red[0];
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(kFinThreads* kFinGroups)
    gate_finalize_kernel(const float* __restrict__ partial, int splits, int B, int N, int heads, int d,
                         const float* __restrict__ t_emb, int E, const float* __restrict__ w_t,
                         const float* __restrict__ w_x, const float* __restrict__ beta, float threshold,
                         float* __restrict__ s_out, float* __restrict__ gate_out) {
  __shared__ float red[kFinThreads];
  __shared__ float grp[kFinGroups][kFinThreads];
  const int bh = blockIdx.x, b = bh / heads, h = bh % heads, t = threadIdx.x;
  const int f = t % kFinThreads, g = t / kFinThreads;
  const size_t C = (size_t)heads * d;
  if (f < d) {
    float sum = 0.f;
    const float* src = partial + (size_t)b * C + (size_t)h * d + f;
#pragma unroll 16
    for (int s = g; s < splits; s += kFinGroups) sum += src[(size_t)s * B * C];
    grp[g][f] = sum;
  }
  __syncthreads();
  float xs = 0.f;
  if (t < d) {
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < kFinGroups; ++i) sum += grp[i][t];
    xs = w_x[(size_t)h * d + t] * (sum / (float)N);
  }
  float ts = 0.f;
  if (t < kFinThreads)
    for (int e = t; e < E; e += kFinThreads) ts = fmaf(w_t[(size_t)h * E + e], t_emb[(size_t)b * E + e], ts);
  const float logit = (block_sum(ts, red) + block_sum(xs, red)) + beta[h];
  if (t == 0) {
    const float sv = 1.0f / (1.0f + expf(-logit));
    if (s_out) s_out[bh] = sv;
    gate_out[bh] = sv < threshold ? 0.0f : sv;
  }
}

}  // namespace

int gate_splits(int B, int N, int* chunk) {
  // about two CTAs per SM over the whole batch, at least 64 tokens each
  const int want = (2 * 148 + B - 1) / B;
  int c = (N + want - 1) / want;
  if (c < 64) c = 64;
  *chunk = c;
  return (N + c - 1) / c;
}

size_t gate_workspace_bytes(int B, int N, int heads, int d) {
  int chunk = 0;
  const int splits = gate_splits(B, N, &chunk);
  return (size_t)splits * B * heads * d * sizeof(float);
}

cudaError_t launch_gate(const GateArgs& a, cudaStream_t s) {
  int chunk = 0;
  const int splits = gate_splits(a.B, a.N, &chunk);
  const int C8 = a.heads * a.d / 8;
  gate_pool_kernel<<<dim3(splits, a.B), dim3(kPoolThreads, kPoolRows), 0, s>>>(
      reinterpret_cast<const uint4*>(a.q), a.N, C8, chunk, a.partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gate_finalize_kernel<<<a.B * a.heads, kFinThreads * kFinGroups, 0, s>>>(
      a.partial, splits, a.B, a.N, a.heads, a.d, a.t_emb, a.E, a.w_t, a.w_x, a.beta, a.threshold, a.s_out, a.gate_out);
  return cudaGetLastError();
}

}  // namespace salad
