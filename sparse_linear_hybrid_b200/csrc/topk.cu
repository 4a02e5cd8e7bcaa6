// Top-K dynamic block mask: the SALAD summary (section 5) says the method also
// applies to Top-K dynamic sparse attention, without a scoring rule.  The rule
// implemented (include/salad.h states it): per (b, h), the mean of q and of k
// over the real tokens of each block; the score of block pair (I, J) is the
// dot product of the two means; query block I keeps the K key blocks with the
// highest scores (ties: the smaller J), listed in ascending J.  The arithmetic
// follows a fixed fp32 order (token sums in token order, one division by the
// token count, an fma chain over the features from 0), so the result is the
// same bit for bit on any implementation that follows it.
//
// topk_pool_kernel    grid (nb, B*Hh), 2*D threads: thread c < D the mean of q
//                     for feature c, thread D + c that of k; CTA (I, bh) also
//                     writes row_ptr (every row has K entries).
// topk_select_kernel  grid (B*Hh, ceil(nb / 16)), 256 threads: the scores of 16
//                     query blocks against every key block (a 16 x 16 thread
//                     tile per chunk of 16 key blocks, means staged in shared
//                     memory), then per row each key block's rank (how many
//                     score better) and the kept ones compacted in order.
// Memory: the pooling reads q and k once (4*d bytes per token per (b, h)); the
// scores are nb^2 * d fused multiply-adds per (b, h).
#include "internal.h"

namespace salad {
namespace {

constexpr int kRows = 16;  // query blocks per selection CTA

template <int D>
__global__ void __launch_bounds__(2 * D) topk_pool_kernel(const uint16_t* __restrict__ q,
                                                          const uint16_t* __restrict__ k, int N, int heads,
                                                          int blk, int nb, int kk, float* __restrict__ qm,
                                                          float* __restrict__ km, int32_t* __restrict__ row_ptr) {
  const int I = blockIdx.x, bh = blockIdx.y, b = bh / heads, h = bh % heads;
  const int t = threadIdx.x;
  const bool is_k = t >= D;
  const int c = is_k ? t - D : t;
  const uint16_t* src = is_k ? k : q;
  const int t0 = I * blk, t1 = min(N, t0 + blk);
  float s = 0.f;
#pragma unroll 8
  for (int tok = t0; tok < t1; ++tok)
    s += __uint_as_float((uint32_t)src[(((size_t)b * N + tok) * heads + h) * D + c] << 16);
  (is_k ? km : qm)[((size_t)bh * nb + I) * D + c] = s / (float)(t1 - t0);
  if (t == 0) {
    const long long r = (long long)bh * nb + I;
    row_ptr[r] = (int32_t)(r * kk);
    if (r == (long long)gridDim.y * nb - 1) row_ptr[r + 1] = (int32_t)((r + 1) * kk);
  }
}

template <int D>
__global__ void __launch_bounds__(256) topk_select_kernel(const float* __restrict__ qm, const float* __restrict__ km,
                                                          int nb, int kk, int32_t* __restrict__ col_idx) {
  extern __shared__ float tk_smem[];
  constexpr int LD = D + 1;  // padded rows: the 16 key-block rows a warp reads sit in different banks
  float* qs = tk_smem;                       // [kRows][LD]
  float* ks = qs + kRows * LD;               // [16][LD]
  float* sc = ks + 16 * LD;                  // [kRows][nb]
  int* keep_flag = reinterpret_cast<int*>(sc + kRows * nb);  // [nb]
  const int bh = blockIdx.x, I0 = blockIdx.y * kRows, tid = threadIdx.x;
  const int nr = min(kRows, nb - I0);
  for (int x = tid; x < nr * D; x += 256) qs[(x / D) * LD + x % D] = qm[((size_t)bh * nb + I0) * D + x];
  const int i = tid / 16, jj = tid % 16;
  for (int J0 = 0; J0 < nb; J0 += 16) {
    const int nj = min(16, nb - J0);
    __syncthreads();
    for (int x = tid; x < nj * D; x += 256) ks[(x / D) * LD + x % D] = km[((size_t)bh * nb + J0) * D + x];
    __syncthreads();
    if (i < nr && jj < nj) {
      float a = 0.f;
#pragma unroll 16
      for (int c = 0; c < D; ++c) a = fmaf(qs[i * LD + c], ks[jj * LD + c], a);
      sc[i * nb + J0 + jj] = a;
    }
  }
  __syncthreads();
  for (int row = 0; row < nr; ++row) {
    const float* srow = sc + row * nb;
    for (int J = tid; J < nb; J += 256) {
      const float v = srow[J];
      int better = 0;
      for (int J2 = 0; J2 < nb; ++J2) {
        const float w = srow[J2];
        better += (w > v || (w == v && J2 < J)) ? 1 : 0;
      }
      keep_flag[J] = better < kk ? 1 : 0;
    }
    __syncthreads();
    int32_t* out = col_idx + ((size_t)bh * nb + I0 + row) * kk;
    for (int J = tid; J < nb; J += 256) {
      if (keep_flag[J]) {
        int pos = 0;
        for (int J2 = 0; J2 < J; ++J2) pos += keep_flag[J2];
        out[pos] = J;
      }
    }
    __syncthreads();
  }
}

template <int D>
cudaError_t launch_topk_t(const TopkArgs& a, cudaStream_t s) {
  const int BH = a.B * a.heads;
  topk_pool_kernel<D><<<dim3(a.nb, BH), 2 * D, 0, s>>>(a.q, a.k, a.N, a.heads, a.block, a.nb, a.kk, a.qm, a.km,
                                                       a.row_ptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(float) * (size_t)(kRows * (D + 1) + 16 * (D + 1) + kRows * a.nb) + sizeof(int) * a.nb;
  e = cudaFuncSetAttribute(topk_select_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  topk_select_kernel<D><<<dim3(BH, (a.nb + kRows - 1) / kRows), 256, smem, s>>>(a.qm, a.km, a.nb, a.kk, a.col_idx);
  return cudaGetLastError();
}

}  // namespace

size_t topk_workspace_bytes(int B, int N, int heads, int d, int block) {
  const size_t nb = ((size_t)N + block - 1) / block;
  return 2 * (size_t)B * heads * nb * d * sizeof(float);
}

cudaError_t launch_topk_mask(const TopkArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_topk_t<64>(a, s) : launch_topk_t<128>(a, s);
}

}  // namespace salad
