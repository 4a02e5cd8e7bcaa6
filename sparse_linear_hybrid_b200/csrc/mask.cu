// Block-mask builder: static spatio-temporal sliding window (ST-SWA) over a
// T x H x W token grid in raster order, reduced to a per-head CSR list of kept
// key blocks (SALAD sparse branch; sciencestack SALAD page, Figure 1 baseline
// "ST-SWA"; SALAD summary section 2.1).
//
// A block of raster-ordered tokens is a union of row segments: each (t, y) row
// it touches contributes one contiguous x interval.  Block pair (I, J) is kept
// iff some segment of I and some segment of J have |dt| <= wt, |dy| <= wh and
// x intervals no more than ww apart.  This is exact for the token-pair rule
// (some i in I, j in J inside the window) because the window is a box.
//
// Three launches: count (one warp per CSR row), an in-place inclusive scan of
// the counts, fill (one warp per row; ballot compaction keeps columns sorted).
// The same kernels build the mask over 3-D tile blocks (bt x bh x bw boxes of
// the grid, numbered in raster order over the boxes).
#include "internal.h"

namespace salad {
namespace {

__device__ __forceinline__ long long llmin(long long a, long long b) { return a < b ? a : b; }

// 3-D tile blocks: box I covers [t0, t0+bt) x [y0, min(H, y0+bh)) x
// [x0, min(W, x0+bw)); two boxes hold a token pair inside the window exactly
// when, on every axis, the gap between their extents is within the window.
__device__ __forceinline__ int axis_gap(int a0, int a1, int b0, int b1) {  // inclusive ranges
  return max(0, max(b0 - a1, a0 - b1));
}

__device__ bool tile_pair_kept(const MaskGrid& g, int wt, int wh, int ww, int I, int J) {
  const int nh = (g.H + g.bh - 1) / g.bh, nw = (g.W + g.bw - 1) / g.bw;
  const int ti = I / (nh * nw), yi = (I / nw) % nh, xi = I % nw;
  const int tj = J / (nh * nw), yj = (J / nw) % nh, xj = J % nw;
  const int ty = axis_gap(ti * g.bt, ti * g.bt + g.bt - 1, tj * g.bt, tj * g.bt + g.bt - 1);
  const int gy = axis_gap(yi * g.bh, min(g.H, yi * g.bh + g.bh) - 1, yj * g.bh, min(g.H, yj * g.bh + g.bh) - 1);
  const int gx = axis_gap(xi * g.bw, min(g.W, xi * g.bw + g.bw) - 1, xj * g.bw, min(g.W, xj * g.bw + g.bw) - 1);
  return ty <= wt && gy <= wh && gx <= ww;
}

__device__ bool block_pair_kept(const MaskGrid& g, int wt, int wh, int ww, int I, int J) {
  if (g.bt > 0) return tile_pair_kept(g, wt, wh, ww, I, J);
  const long long a0 = (long long)I * g.block, a1 = llmin(g.N, a0 + g.block) - 1;
  const long long c0 = (long long)J * g.block, c1 = llmin(g.N, c0 + g.block) - 1;
  const long long ra0 = a0 / g.W, ra1 = a1 / g.W, rc0 = c0 / g.W, rc1 = c1 / g.W;
  // frame-level rejection: the frames of I and J are more than wt apart
  const long long ta0 = ra0 / g.H, ta1 = ra1 / g.H, tc0 = rc0 / g.H, tc1 = rc1 / g.H;
  if (tc0 - ta1 > wt || ta0 - tc1 > wt) return false;
  for (long long ra = ra0; ra <= ra1; ++ra) {
    const int ta = (int)(ra / g.H), ya = (int)(ra % g.H);
    const int xa0 = ra == ra0 ? (int)(a0 % g.W) : 0;
    const int xa1 = ra == ra1 ? (int)(a1 % g.W) : g.W - 1;
    for (long long rc = rc0; rc <= rc1; ++rc) {
      const int tc = (int)(rc / g.H), yc = (int)(rc % g.H);
      if (abs(ta - tc) > wt || abs(ya - yc) > wh) continue;
      const int xc0 = rc == rc0 ? (int)(c0 % g.W) : 0;
      const int xc1 = rc == rc1 ? (int)(c1 % g.W) : g.W - 1;
      const int gap = max(0, max(xc0 - xa1, xa0 - xc1));
      if (gap <= ww) return true;
    }
  }
  return false;
}

// grid (nb, heads), 32 threads: row_ptr[1 + h*nb + I] = number of kept J.
__global__ void __launch_bounds__(32) mask_count_kernel(MaskGrid g, WindowTable win, int32_t* row_ptr) {
  const int I = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  const int wt = win.w[3 * h], wh = win.w[3 * h + 1], ww = win.w[3 * h + 2];
  int cnt = 0;
  for (int J = lane; J < g.nb; J += 32) cnt += block_pair_kept(g, wt, wh, ww, I, J) ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if (lane == 0) row_ptr[1 + (long long)h * g.nb + I] = cnt;
}

// One CTA of 1024 threads: row_ptr[0] = 0, row_ptr[1..n] = inclusive prefix sums.
__global__ void __launch_bounds__(1024) mask_scan_kernel(int32_t* row_ptr, int n) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) {
    carry = 0;
    row_ptr[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += 1024) {
    const int i = base + tid;
    int v = i < n ? row_ptr[1 + i] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    if (warp == 0) {
      int t = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, t, o);
        if (lane >= o) t += u;
      }
      warp_tot[lane] = t;
    }
    __syncthreads();
    const int prefix = carry + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (i < n) row_ptr[1 + i] = prefix + v;
    __syncthreads();
    if (tid == 0) carry += warp_tot[31];
    __syncthreads();
  }
}

// grid (nb, heads), 32 threads: ascending kept columns of row (h, I).
__global__ void __launch_bounds__(32) mask_fill_kernel(MaskGrid g, WindowTable win, const int32_t* row_ptr,
                                                       int32_t* col_idx) {
  const int I = blockIdx.x, h = blockIdx.y, lane = threadIdx.x;
  const int wt = win.w[3 * h], wh = win.w[3 * h + 1], ww = win.w[3 * h + 2];
  int out = row_ptr[(long long)h * g.nb + I];
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int J0 = 0; J0 < g.nb; J0 += 32) {
    const int J = J0 + lane;
    const bool kept = J < g.nb && block_pair_kept(g, wt, wh, ww, I, J);
    const unsigned m = __ballot_sync(0xffffffffu, kept);
    if (kept) col_idx[out + __popc(m & lt_mask)] = J;
    out += __popc(m);
  }
}

}  // namespace

cudaError_t launch_mask_count(const MaskGrid& g, const WindowTable& win, int32_t* row_ptr, cudaStream_t s) {
  mask_count_kernel<<<dim3(g.nb, g.heads), 32, 0, s>>>(g, win, row_ptr);
  return cudaGetLastError();
}

namespace {

// ---------------------------------------------------------------- transpose
// The transposed mask: for every group g (a head, or a (b, h) of a mask with
// rows per (b, h)) and key block J, the ascending query blocks I whose row
// keeps J.  One warp per column (g, J) walks the query blocks 32 at a time and
// tests membership by binary search in each row's ascending list; a ballot
// counts (first pass) or places (second pass) the hits in order, so the result
// is deterministic and needs no sort.
__device__ __forceinline__ bool row_keeps(const int32_t* row_ptr, const int32_t* col_idx, int r, int J) {
  int lo = row_ptr[r], hi = row_ptr[r + 1];  // [lo, hi)
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    const int c = col_idx[mid];
    if (c == J) return true;
    if (c < J) {
      lo = mid + 1;
    } else {
      hi = mid;
    }
  }
  return false;
}

template <bool FILL>
__global__ void __launch_bounds__(128) mask_t_kernel(const int32_t* __restrict__ row_ptr,
                                                     const int32_t* __restrict__ col_idx, int nb,
                                                     int32_t* __restrict__ t_row_ptr, int32_t* __restrict__ t_col_idx,
                                                     uint32_t* status) {
  const int lane = threadIdx.x & 31;
  const int J = blockIdx.x * 4 + (threadIdx.x >> 5), g = blockIdx.y;
  if (J >= nb) return;
  const int rows = (int)gridDim.y * nb;
  int pos = FILL ? t_row_ptr[(size_t)g * nb + J] : 0;
  for (int I0 = 0; I0 < nb; I0 += 32) {
    const int I = I0 + lane;
    // (debug builds: a row whose range is malformed is searched as empty)
    const bool has = I < nb && debug_row_ok(row_ptr, col_idx, g * nb + I, rows, nb, false, status) &&
                     row_keeps(row_ptr, col_idx, g * nb + I, J);
    const uint32_t m = __ballot_sync(0xffffffffu, has);
    if (FILL && has) t_col_idx[pos + __popc(m & ((1u << lane) - 1u))] = I;
    pos += __popc(m);
  }
  if (!FILL && lane == 0) t_row_ptr[(size_t)g * nb + J + 1] = pos;  // counts, then the scan
}

}  // namespace

cudaError_t launch_mask_transpose(const int32_t* row_ptr, const int32_t* col_idx, int groups, int nb,
                                  int32_t* t_row_ptr, int32_t* t_col_idx, uint32_t* status, cudaStream_t s) {
  const dim3 grid((nb + 3) / 4, groups);
  mask_t_kernel<false><<<grid, 128, 0, s>>>(row_ptr, col_idx, nb, t_row_ptr, nullptr, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mask_scan_kernel<<<1, 1024, 0, s>>>(t_row_ptr, groups * nb);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  mask_t_kernel<true><<<grid, 128, 0, s>>>(row_ptr, col_idx, nb, t_row_ptr, t_col_idx, status);
  return cudaGetLastError();
}

cudaError_t launch_mask_scan(int32_t* row_ptr, int n, cudaStream_t s) {
  mask_scan_kernel<<<1, 1024, 0, s>>>(row_ptr, n);
  return cudaGetLastError();
}

cudaError_t launch_mask_fill(const MaskGrid& g, const WindowTable& win, const int32_t* row_ptr, int32_t* col_idx,
                             cudaStream_t s) {
  mask_fill_kernel<<<dim3(g.nb, g.heads), 32, 0, s>>>(g, win, row_ptr, col_idx);
  return cudaGetLastError();
}

}  // namespace salad
