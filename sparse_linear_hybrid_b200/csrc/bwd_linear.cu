// Backward pass of the linear branch, its projection and the gate (the rest of
// the layer's gradients next to the sparse branch's in bwd.cu).  Per (b, h),
// with S and z the branch's state, a_i = relu(q_i), den_i = a_i.z + eps,
// o_i = a_i^T S / den_i, y_i = o_i W and G = dL/dout:
//   dgate      = sum_i G_i.y_i
//   dy_i       = g G_i,  dW += sum_i o_i^T dy_i  (over every (b, h))
//   do_i       = dy_i W^T,  du_i = do_i / den_i,  dden_i = -(do_i.o_i) / den_i
//   dS         = sum_i a_i du_i^T,   dz = sum_i dden_i a_i
//   dq_i      += [q_i > 0] (S du_i + dden_i z)
//   dk_j      += [k_j > 0] (dS v_j + dz),   dv_j += dS^T relu(k_j)
// and, for the sparse branch, D_i = G_i.(out_i - g y_i) (its output is out
// minus the linear term).  fp32 CUDA-core arithmetic in a fixed order:
//   lin_rows_kernel    per 128 query rows of a (b, h), one thread per feature,
//                      S, S^T, W, W^T in shared memory: the per-row terms; it
//                      writes dq (the sparse backward then adds its part), D_i,
//                      lse_i in base 2, and o, dy, du, dden, G.y for the sums
//   lin_outer_kernel   split sums of a_i du_i^T (dS) and o_i dy_i^T (dW), 16 x 16
//                      threads each owning a block of the d x d result
//   lin_vec_kernel     dz and dgate per (b, h): eight row groups, added in order
//   lin_reduce_kernel  the splits (and, for dW, the (b, h)) in order
//   lin_keys_kernel    per 128 key rows: the linear parts of dk and dv
#include "internal.h"
#include "ptx.cuh"

namespace salad {
namespace {

constexpr int kOuterThreads = 256;
constexpr int kOuterRows = 32;  // rows staged per step of lin_outer_kernel
constexpr int kVecGroups = 8;
constexpr float kLog2eL = 1.4426950408889634f;

__device__ __forceinline__ float bf16f(uint16_t x) { return __uint_as_float((uint32_t)x << 16); }

// Fixed-order tree sum over the D threads of the block.
template <int D>
__device__ float tree_sum(float v, float* red) {
  red[threadIdx.x] = v;
  __syncthreads();
#pragma unroll
  for (int s = D / 2; s > 0; s >>= 1) {
    if ((int)threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  const float r = red[0];
  __syncthreads();
  return r;
}

template <int D>
__global__ void __launch_bounds__(D) lin_rows_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ out,
                                                     const uint16_t* __restrict__ dout, const float* __restrict__ lse,
                                                     const uint16_t* __restrict__ w, const float* __restrict__ gate,
                                                     const float* __restrict__ S, const float* __restrict__ z, int N,
                                                     int heads, int npad, float eps, float* __restrict__ dq,
                                                     float* __restrict__ lse2, float* __restrict__ dvec,
                                                     float* __restrict__ o_s, float* __restrict__ dy_s,
                                                     float* __restrict__ du_s, float* __restrict__ dden_s,
                                                     float* __restrict__ yg_s) {
  extern __shared__ float lin_smem[];
  float* Ss = lin_smem;            // [D][D]: S[c][e]
  float* St = Ss + D * D;          // [D][D]: S[e][c]
  uint16_t* Ws = reinterpret_cast<uint16_t*>(St + D * D);  // [D][D] bf16: W[e][f]
  uint16_t* Wt = Ws + D * D;                                // [D][D] bf16: W[f][e]
  float* zs = reinterpret_cast<float*>(Wt + D * D);         // [D]
  float* a = zs + D;               // [D] per row
  float* o = a + D;
  float* dy = o + D;
  float* du = dy + D;
  float* red = du + D;
  const int t = threadIdx.x, bh = blockIdx.y, b = bh / heads, h = bh % heads;
  const float g = gate[bh];
  for (int x = t; x < D * D; x += D) {
    const int r = x / D, c = x % D;
    const float sv = S[(size_t)bh * D * D + x];
    Ss[x] = sv;
    St[c * D + r] = sv;
    Ws[x] = w[x];
    Wt[c * D + r] = w[x];
  }
  zs[t] = z[(size_t)bh * D + t];
  __syncthreads();
  const int r0 = blockIdx.x * 128, r1 = min(N, r0 + 128);
  for (int i = r0; i < r1; ++i) {
    const size_t off = (((size_t)b * N + i) * heads + h) * D;
    const size_t ri = (size_t)bh * N + i;
    const float qv = bf16f(q[off + t]);
    const float Gt = bf16f(dout[off + t]);
    a[t] = qv > 0.f ? qv : 0.f;
    __syncthreads();
    const float den = eps + tree_sum<D>(a[t] * zs[t], red);
    float u = 0.f;
#pragma unroll 8
    for (int c = 0; c < D; ++c) u = fmaf(a[c], Ss[c * D + t], u);
    const float ot = u / den;
    o[t] = ot;
    __syncthreads();
    float y = 0.f;
#pragma unroll 8
    for (int e = 0; e < D; ++e) y = fmaf(o[e], bf16f(Ws[e * D + t]), y);
    const float yg = tree_sum<D>(Gt * y, red);
    const float Dval = tree_sum<D>(Gt * (bf16f(out[off + t]) - g * y), red);
    dy[t] = g * Gt;
    __syncthreads();
    float dov = 0.f;
#pragma unroll 8
    for (int f = 0; f < D; ++f) dov = fmaf(bf16f(Wt[f * D + t]), dy[f], dov);
    const float dden = -tree_sum<D>(dov * ot, red) / den;
    du[t] = dov / den;
    __syncthreads();
    float dA = dden * zs[t];
#pragma unroll 8
    for (int e = 0; e < D; ++e) dA = fmaf(St[e * D + t], du[e], dA);
    dq[off + t] = qv > 0.f ? dA : 0.f;
    o_s[off + t] = ot;
    dy_s[off + t] = dy[t];
    du_s[off + t] = du[t];
    if (t == 0) {
      dden_s[ri] = dden;
      yg_s[ri] = yg;
      dvec[(size_t)bh * npad + i] = Dval;
      lse2[(size_t)bh * npad + i] = lse[ri] * kLog2eL;
    }
    __syncthreads();
  }
  // pad rows of the last tile: no probability mass, no D
  if (blockIdx.x == gridDim.x - 1)
    for (int i = N + t; i < npad; i += D) {
      lse2[(size_t)bh * npad + i] = INFINITY;
      dvec[(size_t)bh * npad + i] = 0.f;
    }
}

// Split sums of x_i y_i^T over the rows of a split: product 0 is
// relu(q_i) du_i^T (dS), product 1 is o_i dy_i^T (dW); fp32 partials
// [2][splits][B*Hh][D][D].
template <int D>
__global__ void __launch_bounds__(kOuterThreads) lin_outer_kernel(const uint16_t* __restrict__ q,
                                                                  const float* __restrict__ o_s,
                                                                  const float* __restrict__ dy_s,
                                                                  const float* __restrict__ du_s, int N, int heads,
                                                                  int rows_per_split, float* __restrict__ partial) {
  constexpr int M = D / 16;  // the M x M block of the result each thread owns
  __shared__ float xs[kOuterRows][D];
  __shared__ float ys[kOuterRows][D];
  const int split = blockIdx.x, bh = blockIdx.y, prod = blockIdx.z, b = bh / heads, h = bh % heads;
  const int ti = threadIdx.x / 16, tj = threadIdx.x % 16;
  float acc[M][M];
#pragma unroll
  for (int i = 0; i < M; ++i)
#pragma unroll
    for (int j = 0; j < M; ++j) acc[i][j] = 0.f;
  const int n0 = split * rows_per_split, n1 = min(N, n0 + rows_per_split);
  for (int c0 = n0; c0 < n1; c0 += kOuterRows) {
    const int nr = min(kOuterRows, n1 - c0);
    for (int x = threadIdx.x; x < kOuterRows * D; x += kOuterThreads) {
      const int r = x / D, f = x % D;
      float xv = 0.f, yv = 0.f;
      if (r < nr) {
        const size_t off = (((size_t)b * N + c0 + r) * heads + h) * D + f;
        if (prod == 0) {
          const float qv = bf16f(q[off]);
          xv = qv > 0.f ? qv : 0.f;
          yv = du_s[off];
        } else {
          xv = o_s[off];
          yv = dy_s[off];
        }
      }
      xs[r][f] = xv;
      ys[r][f] = yv;
    }
    __syncthreads();
    for (int r = 0; r < nr; ++r) {
      float xr[M], yr[M];
#pragma unroll
      for (int i = 0; i < M; ++i) {
        xr[i] = xs[r][ti * M + i];
        yr[i] = ys[r][tj * M + i];
      }
#pragma unroll
      for (int i = 0; i < M; ++i)
#pragma unroll
        for (int j = 0; j < M; ++j) acc[i][j] = fmaf(xr[i], yr[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* dst = partial + (((size_t)prod * gridDim.x + split) * gridDim.y + bh) * D * D;
#pragma unroll
  for (int i = 0; i < M; ++i)
#pragma unroll
    for (int j = 0; j < M; ++j) dst[(ti * M + i) * D + tj * M + j] = acc[i][j];
}

// dz[bh][c] = sum_i dden_i relu(q_ic) and dgate[bh] = sum_i yg_i: eight groups of
// D threads take every eighth row, the groups are added in order.
template <int D>
__global__ void __launch_bounds__(D * kVecGroups) lin_vec_kernel(const uint16_t* __restrict__ q,
                                                                 const float* __restrict__ dden_s,
                                                                 const float* __restrict__ yg_s, int N, int heads,
                                                                 float* __restrict__ dz, float* __restrict__ dgate) {
  __shared__ float gz[kVecGroups][D];
  __shared__ float gg[kVecGroups];
  const int bh = blockIdx.x, b = bh / heads, h = bh % heads;
  const int c = threadIdx.x % D, grp = threadIdx.x / D;
  float acc = 0.f, accg = 0.f;
#pragma unroll 4
  for (int i = grp; i < N; i += kVecGroups) {
    const float qv = bf16f(q[(((size_t)b * N + i) * heads + h) * D + c]);
    const float dd = dden_s[(size_t)bh * N + i];
    if (qv > 0.f) acc = fmaf(dd, qv, acc);
    if (c == 0) accg += yg_s[(size_t)bh * N + i];
  }
  gz[grp][c] = acc;
  if (c == 0) gg[grp] = accg;
  __syncthreads();
  if (grp == 0) {
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < kVecGroups; ++k) s += gz[k][c];
    dz[(size_t)bh * D + c] = s;
    if (c == 0) {
      float sg = 0.f;
#pragma unroll
      for (int k = 0; k < kVecGroups; ++k) sg += gg[k];
      dgate[bh] = sg;
    }
  }
}

// dS[bh] = the splits of product 0 in order; dW = product 1 over the splits of
// each (b, h) in order, the (b, h) in order.
template <int D>
__global__ void __launch_bounds__(256) lin_reduce_kernel(const float* __restrict__ partial, int splits, int BH,
                                                         float* __restrict__ dS, float* __restrict__ dw) {
  const int e = blockIdx.x * 256 + threadIdx.x;
  if (e >= D * D) return;
  const int bh = blockIdx.y;
  if (bh < BH) {
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += partial[(((size_t)0 * splits + k) * BH + bh) * D * D + e];
    dS[(size_t)bh * D * D + e] = s;
  } else {
    float s = 0.f;
    for (int x = 0; x < BH; ++x) {
      float sb = 0.f;
      for (int k = 0; k < splits; ++k) sb += partial[(((size_t)1 * splits + k) * BH + x) * D * D + e];
      s += sb;
    }
    dw[e] = s;
  }
}

// The linear parts of dk and dv for 128 key rows of a (b, h), added to the
// sparse branch's.
template <int D>
__global__ void __launch_bounds__(D) lin_keys_kernel(const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
                                                     const float* __restrict__ dS, const float* __restrict__ dz, int N,
                                                     int heads, float* __restrict__ dk, float* __restrict__ dv) {
  extern __shared__ float lin_smem[];
  float* Ds = lin_smem;      // [D][D]: dS[c][e]
  float* Dt = Ds + D * D;    // [D][D]: dS[e][c]
  float* kr = Dt + D * D;    // [D] relu(k_j)
  float* vr = kr + D;        // [D] v_j
  const int t = threadIdx.x, bh = blockIdx.y, b = bh / heads, h = bh % heads;
  for (int x = t; x < D * D; x += D) {
    const float sv = dS[(size_t)bh * D * D + x];
    Ds[x] = sv;
    Dt[(x % D) * D + x / D] = sv;
  }
  const float dzt = dz[(size_t)bh * D + t];
  __syncthreads();
  const int r0 = blockIdx.x * 128, r1 = min(N, r0 + 128);
  for (int j = r0; j < r1; ++j) {
    const size_t off = (((size_t)b * N + j) * heads + h) * D;
    const float kv = bf16f(k[off + t]);
    kr[t] = kv > 0.f ? kv : 0.f;
    vr[t] = bf16f(v[off + t]);
    __syncthreads();
    float tk = dzt, tv = 0.f;
#pragma unroll 8
    for (int e = 0; e < D; ++e) {
      tk = fmaf(Dt[e * D + t], vr[e], tk);  // (dS v_j)_t
      tv = fmaf(Ds[e * D + t], kr[e], tv);  // (dS^T relu(k_j))_t
    }
    if (kv > 0.f) dk[off + t] += tk;
    dv[off + t] += tv;
    __syncthreads();
  }
}

template <int D>
cudaError_t launch_lin_rows_t(const LinBwdArgs& a, cudaStream_t s) {
  const size_t smem = (size_t)(2 * D * D + 6 * D) * sizeof(float) + (size_t)2 * D * D * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(lin_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  lin_rows_kernel<D><<<dim3(a.npad / 128, a.B * a.heads), D, smem, s>>>(
      a.q, a.out, a.dout, a.lse, a.w, a.gate, a.S, a.z, a.N, a.heads, a.npad, a.eps, a.dq, a.lse2, a.dvec, a.o_s,
      a.dy_s, a.du_s, a.dden_s, a.yg_s);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_lin_tail_t(const LinBwdArgs& a, cudaStream_t s) {
  const int BH = a.B * a.heads;
  const int rps = (a.N + a.splits - 1) / a.splits;
  lin_outer_kernel<D><<<dim3(a.splits, BH, 2), kOuterThreads, 0, s>>>(a.q, a.o_s, a.dy_s, a.du_s, a.N, a.heads, rps,
                                                                     a.partial);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  lin_vec_kernel<D><<<BH, D * kVecGroups, 0, s>>>(a.q, a.dden_s, a.yg_s, a.N, a.heads, a.dz, a.dgate);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lin_reduce_kernel<D><<<dim3((D * D + 255) / 256, BH + 1), 256, 0, s>>>(a.partial, a.splits, BH, a.dS, a.dw);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t smem = (size_t)(2 * D * D + 2 * D) * sizeof(float);
  if ((e = cudaFuncSetAttribute(lin_keys_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  lin_keys_kernel<D><<<dim3(a.npad / 128, BH), D, smem, s>>>(a.k, a.v, a.dS, a.dz, a.N, a.heads, a.dk, a.dv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_linear_backward_rows(const LinBwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_lin_rows_t<64>(a, s) : launch_lin_rows_t<128>(a, s);
}

cudaError_t launch_linear_backward_tail(const LinBwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_lin_tail_t<64>(a, s) : launch_lin_tail_t<128>(a, s);
}

}  // namespace salad
