// Backward pass of the sparse branch (block-sparse softmax attention over the
// kept key blocks; the fine-tuning of the SALAD summary, section 3, trains
// through it).  With p_ij = exp(scale q_i.k_j - lse_i) over the kept keys,
// the row log-sum-exp lse_i kept by the forward, and o_i the branch output:
//   D_i   = dout_i . o_i
//   dp_ij = dout_i . v_j,      ds_ij = p_ij (dp_ij - D_i)
//   dq_i  = scale sum_j ds_ij k_j
//   dk_j  = scale sum_i ds_ij q_i,      dv_j = sum_i p_ij dout_i
// Three kernels (raster blocks of 128 tokens):
//   bwd_prep_kernel  D_i and lse_i in base 2 (lse * log2 e) into the workspace,
//                    rows padded to whole 128-row tiles (pad rows: p = 0, D = 0)
//   bwd_dq_kernel    one CTA per (query tile, b, h), over its kept key tiles:
//                    S = Q K^T and dP = dO V^T on the tensor cores (SS form),
//                    one thread per row forms dS = P (dP - D) into tensor
//                    memory as bf16, and dQ += dS K (A from tensor memory, K
//                    as an MN-major B operand)
//   bwd_dkdv_kernel  one CTA per (key tile, b, h), over the query tiles whose
//                    rows keep it (the transposed mask): S^T = K Q^T and
//                    dP^T = V dO^T, one thread per key row forms P^T and dS^T
//                    (bf16, written over the columns of S^T it has read),
//                    dV += P^T dO and dK += dS^T Q.  dP^T of the next tile
//                    runs as soon as dP^T is in the row warps' registers, and
//                    the products of the first query half while the row warps
//                    form the second.
// Warp roles, 320 threads: warp 0 lane 0 issues the TMA loads and the MMAs in
// program order (K/V or Q/dO tiles in a 2-deep ring), warp 1 owns the tensor
// memory, warps 2-9 take one row each (TMEM lane quarter = warp % 4) and 64 of
// its 128 columns (warp (w - 2) / 4 picks which); the exponentials of one pair
// in four run on the FMA pipe (exp2_fma_x2), the rest on the MUFU.  Every
// barrier wait is bounded; on a time-out the kernel records it and drains.
// Gradients are written in fp32.
#include "internal.h"
#include "ptx.cuh"

namespace salad {
namespace {

constexpr int kBwdThreads = 320;  // producer/issuer, TMEM owner, eight row warps
constexpr uint64_t kBwdDrainNs = 1000000000ull;
constexpr float kLog2e = 1.4426950408889634f;

struct BwdShared {
  uint64_t fixed_full;    // the CTA's fixed tiles (Q and dO, or K and V)
  uint64_t ring_full[2];  // dK/dV kernel: the streamed tiles (Q, dO and the row vectors)
  uint64_t k_full[3];     // dQ kernel: the K ring (three stages)
  uint64_t v_full[2];     // dQ kernel: the V ring (two stages)
  uint64_t dp_full;       // dP (dQ kernel) or dP^T (dK/dV kernel) of the current tile is in tensor memory
  uint64_t s_full;        // S (dQ kernel) or S^T (dK/dV kernel) of the current tile is in tensor memory
  uint64_t s_read;        // dQ kernel: the row warps have read S of the current tile
  uint64_t dp_read;       // dK/dV kernel: the row warps have read dP^T of the current tile
  uint64_t ds_h[2];       // dK/dV kernel: P^T and dS^T of one query half of the current tile are written
  uint64_t grads_done;    // dK/dV kernel: the gradient products of the last tile have completed
  uint64_t ds_full;       // dQ kernel: the eight row warps have written dS of the tile
  uint64_t mm_done;       // the gradient products of the tile have completed
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

template <int D>
struct BwdCfg {
  static constexpr int DCH = D / 64;
  static constexpr int TILE = 128 * D * 2;  // one 128-row tile of q, k, v or dout (DCH boxes of 16 KB)
  static constexpr int VEC = 2 * 128 * 4;   // lse2 and D of 128 rows
  static constexpr int OFF_FIX = 0;         // two fixed tiles
  static constexpr int OFF_RING = 2 * TILE; // two stages of two tiles
  static constexpr int OFF_VEC = 6 * TILE;  // two stages of row vectors (dK/dV kernel)
  static constexpr int OFF_BAR = OFF_VEC + 2 * VEC;
  static constexpr int SMEM_USED = OFF_BAR + (int)sizeof(BwdShared) + 1024;
  // at least 120 KB so that one CTA (and its 512 TMEM columns) owns the SM
  static constexpr int SMEM = SMEM_USED > 122880 ? SMEM_USED : 122880;
  // dQ kernel: Q and dO, then a three-stage K ring and a two-stage V ring (K_j is
  // read by S_j and the dQ product, V_j only by dP_j, which completes earlier)
  static constexpr int DQ_OFF_K = 2 * TILE;
  static constexpr int DQ_OFF_V = 5 * TILE;
  static constexpr int DQ_OFF_BAR = 7 * TILE;
  static constexpr int DQ_SMEM = DQ_OFF_BAR + (int)sizeof(BwdShared) + 1024;
  static constexpr uint32_t IDESC_SS = idesc_bf16(128, 128, false, false);  // X Y^T, both K-major
  static constexpr uint32_t IDESC_G = idesc_bf16(128, D, false, true);      // A (tmem) x B (MN-major)
  static_assert(SMEM <= 232448 && DQ_SMEM <= 232448, "shared memory budget");
};

// 128 x 128 product X Y^T of two K-major 128 x D tiles in shared memory.
template <int D>
__device__ __forceinline__ void mma_xyt(uint32_t d_tmem, uint32_t x, uint32_t y) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const uint32_t off = (kk / 4) * 16384 + (kk % 4) * 32;
    mma_bf16_ss(d_tmem, sw128_desc(x + off, 16, 1024), sw128_desc(y + off, 16, 1024), BwdCfg<D>::IDESC_SS,
                kk > 0 ? 1u : 0u);
  }
}

// 128 x 128 product X Y^T with X (128 x D bf16) in tensor memory from column
// x_tmem and Y a K-major 128 x D tile in shared memory: one shared operand per
// MMA instead of two.
template <int D>
__device__ __forceinline__ void mma_tyt(uint32_t d_tmem, uint32_t x_tmem, uint32_t y) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    mma_bf16_ts(d_tmem, x_tmem + kk * 8, sw128_desc(y + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024),
                BwdCfg<D>::IDESC_SS, kk > 0 ? 1u : 0u);
}

// A 128 x D bf16 tile of shared memory (K-major, 128-byte swizzle) into tensor
// memory columns [t, t + D / 2): row i to lane i; ordered with the MMAs issued
// later by the same thread.
template <int D>
__device__ __forceinline__ void copy_tile_to_tmem(uint32_t t, uint32_t tile) {
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
    tmem_cp_128x256b(t + kk * 8, sw128_desc(tile + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024));
}

// D += A B with A = 128 x 128 bf16 in tensor memory, B a 128 x D tile in shared
// memory read as an MN-major operand.  A's K = 128 pairs of columns sit at
// a_tmem + [0, 64) (split = false) or, written by two column halves each into
// its own range, at a_tmem + [0, 32) and a_tmem + [64, 96) (split = true).
template <int D>
__device__ __forceinline__ void mma_grad(uint32_t d_tmem, uint32_t a_tmem, uint32_t b, bool accumulate,
                                         bool split) {
#pragma unroll
  for (int kk = 0; kk < 8; ++kk) {
    const uint32_t a = a_tmem + (split && kk >= 4 ? 64 + (kk - 4) * 8 : kk * 8);
    mma_bf16_ts(d_tmem, a, sw128_desc(b + kk * 2048, 16384, 1024), BwdCfg<D>::IDESC_G,
                (accumulate || kk > 0) ? 1u : 0u);
  }
}

// D += A_h B_h over query half h of a tile (dK/dV kernel): A_h = 128 x 64 bf16 in
// tensor memory, its K = 64 query columns packed in pairs at a_tmem + [0, 16)
// (queries [0, 32) of the half) and a_tmem + [32, 48) (queries [32, 64)); B_h =
// rows [64 h, 64 h + 64) of a 128 x D tile in shared memory read as an MN-major
// operand (b_half = B + 8192 h).
template <int D>
__device__ __forceinline__ void mma_grad_half(uint32_t d_tmem, uint32_t a_tmem, uint32_t b_half, bool accumulate) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
    mma_bf16_ts(d_tmem, a_tmem + 32 * (kk >> 1) + 8 * (kk & 1), sw128_desc(b_half + kk * 2048, 16384, 1024),
                BwdCfg<D>::IDESC_G, (accumulate || kk > 0) ? 1u : 0u);
}

// p = 2^(s * c - l) for the 32 values of a row chunk, 0 from column `valid` on;
// one pair in four on the FMA pipe.
__device__ __forceinline__ void exp_chunk(const uint32_t (&sr)[32], float c, float l, int col0, int valid,
                                          float* p) {
  const uint64_t c2 = f32x2_pack(c, c), nl = f32x2_pack(-l, -l);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const uint64_t x = f32x2_fma(f32x2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, nl);
    float p0, p1;
    if ((i & 3) == 3) {
      exp2_fma_x2(x, p0, p1);
    } else {
      float x0, x1;
      f32x2_unpack(x, x0, x1);
      p0 = ex2_approx(x0);
      p1 = ex2_approx(x1);
    }
    p[2 * i] = col0 + 2 * i < valid ? p0 : 0.f;
    p[2 * i + 1] = col0 + 2 * i + 1 < valid ? p1 : 0.f;
  }
}

__device__ __forceinline__ void bwd_timeout(BwdShared* sh, uint32_t* status) {
  sh->abort_flag = 1;
  atomicOr(status, kStatusTimeout);
}

// D_i and lse_i * log2 e per row, into [B*Hh][Npad] (pad rows: lse2 = +inf, D = 0).
template <int D>
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const uint16_t* __restrict__ o, const uint16_t* __restrict__ dout, const float* __restrict__ lse,
                    int B, int N, int heads, int npad, float* __restrict__ lse2, float* __restrict__ dvec) {
  const long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= (long long)B * heads * npad) return;
  const int bh = (int)(t / npad), n = (int)(t % npad), b = bh / heads, h = bh % heads;
  if (n >= N) {
    lse2[t] = INFINITY;
    dvec[t] = 0.f;
    return;
  }
  const uint4* po = reinterpret_cast<const uint4*>(o + (((size_t)b * N + n) * heads + h) * D);
  const uint4* pd = reinterpret_cast<const uint4*>(dout + (((size_t)b * N + n) * heads + h) * D);
  float acc = 0.f;
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const uint4 x = po[c], y = pd[c];
    const uint32_t xa[4] = {x.x, x.y, x.z, x.w}, ya[4] = {y.x, y.y, y.z, y.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc = fmaf(bf16_lo_to_f32(xa[i]), bf16_lo_to_f32(ya[i]), acc);
      acc = fmaf(bf16_hi_to_f32(xa[i]), bf16_hi_to_f32(ya[i]), acc);
    }
  }
  dvec[t] = acc;
  lse2[t] = lse[(size_t)bh * N + n] * kLog2e;
}

// ------------------------------------------------------------------ dQ
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                  const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                  const float* __restrict__ lse2, const float* __restrict__ dvec, float* __restrict__ dq, int N,
                  int heads, int nb, int npad, int mask_per_bh, float scale, float scale_log2, uint32_t* status,
                  uint64_t limit_ns, int accumulate) {
  using C = BwdCfg<D>;
  // S [0,128), dP [128,256) (dS as bf16 over its own dP: columns [0,32) and
  // [64,96), one range per column half), dQ [256,256+D), then Q and dO as bf16
  // A operands: [384,384+D/2) and [448,448+D/2)
  constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DQ = 256, TM_Q = 384, TM_DO = 448;
  extern __shared__ uint8_t bwd_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bwd_smem_raw) + 1023) & ~uintptr_t(1023));
  BwdShared* sh = reinterpret_cast<BwdShared*>(smem + C::DQ_OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x % nb, bh = blockIdx.x / nb, b = bh / heads, h = bh % heads;
  const int mrow = (mask_per_bh ? bh : h) * nb + qt;
  const int mask_rows = (mask_per_bh ? (int)(gridDim.x / nb) : heads) * nb;
  const int c0 = row_ptr[mrow];
  const int n = debug_row_ok(row_ptr, col_idx, mrow, mask_rows, nb, true, status) ? row_ptr[mrow + 1] - c0 : 0;

  if (threadIdx.x == 0) {
    mbar_init(&sh->fixed_full, 1);
    for (int st = 0; st < 3; ++st) mbar_init(&sh->k_full[st], 1);
    for (int st = 0; st < 2; ++st) mbar_init(&sh->v_full[st], 1);
    mbar_init(&sh->dp_full, 1);
    mbar_init(&sh->s_full, 1);
    mbar_init(&sh->s_read, 8);
    mbar_init(&sh->ds_full, 8);
    mbar_init(&sh->mm_done, 1);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t q_s = sbase + C::OFF_FIX, do_s = q_s + C::TILE;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int kl = 0, vl = 0;  // K and V loads issued
      auto load_k = [&](int j) {
        const int st = j % 3, col = col_idx[c0 + j];
        mbar_arrive_expect_tx(&sh->k_full[st], C::TILE);
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          tma_load_3d(smem + C::DQ_OFF_K + st * C::TILE + ch * 16384, &tm_k, &sh->k_full[st], h * D + ch * 64,
                      col * 128, b);
        ++kl;
      };
      auto load_v = [&](int j) {
        const int st = j & 1, col = col_idx[c0 + j];
        mbar_arrive_expect_tx(&sh->v_full[st], C::TILE);
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          tma_load_3d(smem + C::DQ_OFF_V + st * C::TILE + ch * 16384, &tm_v, &sh->v_full[st], h * D + ch * 64,
                      col * 128, b);
        ++vl;
      };
      auto k_tile = [&](int j) { return sbase + C::DQ_OFF_K + (j % 3) * C::TILE; };
      auto v_tile = [&](int j) { return sbase + C::DQ_OFF_V + (j & 1) * C::TILE; };
      auto wait_k = [&](int j) { return mbar_wait(&sh->k_full[j % 3], (uint32_t)((j / 3) & 1), limit_ns); };
      auto wait_v = [&](int j) { return mbar_wait(&sh->v_full[j & 1], (uint32_t)((j >> 1) & 1), limit_ns); };
      mbar_arrive_expect_tx(&sh->fixed_full, 2 * C::TILE);
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch) {
        tma_load_3d(smem + C::OFF_FIX + ch * 16384, &tm_q, &sh->fixed_full, h * D + ch * 64, qt * 128, b);
        tma_load_3d(smem + C::OFF_FIX + C::TILE + ch * 16384, &tm_do, &sh->fixed_full, h * D + ch * 64, qt * 128,
                    b);
      }
      for (int j = 0; j < n && j < 3; ++j) load_k(j);
      for (int j = 0; j < n && j < 2; ++j) load_v(j);
      // Q and dO go to tensor memory once, so that S = Q K^T and dP = dO V^T read
      // one shared operand each.  Schedule: S_{j+1} as soon as the row warps have
      // read S_j (while they form dS_j over dP_j), then dQ += dS_j K_j and
      // dP_{j+1} (after the dQ product, in issue order) while they take the
      // exponentials of S_{j+1}.  K_{j+3} refills K_j's stage once the dQ product
      // has read it, V_{j+2} refills V_j's once dP_j is done.
      ok = mbar_wait(&sh->fixed_full, 0, limit_ns);
      if (ok && n >= 1) {
        ok = wait_k(0) && wait_v(0);
        if (ok) {
          tc_fence_after();
          copy_tile_to_tmem<D>(tmem + TM_Q, q_s);
          copy_tile_to_tmem<D>(tmem + TM_DO, do_s);
          mma_tyt<D>(tmem + TM_S, tmem + TM_Q, k_tile(0));
          mma_commit(&sh->s_full);
          mma_tyt<D>(tmem + TM_DP, tmem + TM_DO, v_tile(0));
          mma_commit(&sh->dp_full);
        }
      }
      for (int j = 0; ok && j < n; ++j) {
        if (j + 1 < n) {
          // S_{j+1} over S_j once the row warps have read it
          if (sh->abort_flag || !mbar_wait(&sh->s_read, (uint32_t)(j & 1), limit_ns) || !wait_k(j + 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_tyt<D>(tmem + TM_S, tmem + TM_Q, k_tile(j + 1));
          mma_commit(&sh->s_full);
        }
        if (sh->abort_flag || !mbar_wait(&sh->ds_full, (uint32_t)(j & 1), limit_ns)) { ok = false; break; }
        tc_fence_after();
        mma_grad<D>(tmem + TM_DQ, tmem + TM_DP, k_tile(j), j > 0, true);
        mma_commit(&sh->mm_done);
        // dP_j completed before the row warps formed dS_j: V_j's stage is free
        if (j + 2 < n) load_v(j + 2);
        if (j + 1 < n) {
          // dP_{j+1} over dS_j, after the dQ product that reads it (issue order)
          if (!wait_v(j + 1)) { ok = false; break; }
          tc_fence_after();
          mma_tyt<D>(tmem + TM_DP, tmem + TM_DO, v_tile(j + 1));
          mma_commit(&sh->dp_full);
        }
        if (j + 3 < n) {
          // K_j's stage is free once the dQ product of tile j has read it
          if (!mbar_wait(&sh->mm_done, (uint32_t)(j & 1), limit_ns)) { ok = false; break; }
          load_k(j + 3);
        }
      }
      if (!ok) {
        bwd_timeout(sh, status);
        mma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kBwdDrainNs);
      }
      // every copy this thread started lands before the CTA exits
      mbar_wait(&sh->fixed_full, 0, kBwdDrainNs);
      for (int i = (kl > 3 ? kl - 3 : 0); i < kl; ++i)
        mbar_wait(&sh->k_full[i % 3], (uint32_t)((i / 3) & 1), kBwdDrainNs);
      for (int i = (vl > 2 ? vl - 2 : 0); i < vl; ++i)
        mbar_wait(&sh->v_full[i & 1], (uint32_t)((i >> 1) & 1), kBwdDrainNs);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- one thread per query row
    // and column half: keys [64 half, 64 half + 64) of each key tile
    const int quarter = warp & 3, r = quarter * 32 + lane, half = (warp - 2) >> 2;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const float l2 = lse2[(size_t)bh * npad + qt * 128 + r];
    const float Dr = dvec[(size_t)bh * npad + qt * 128 + r];
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int valid = min(128, N - col_idx[c0 + j] * 128);  // real keys of the tile
      // P of the row from S_j (fp32, kept in registers), then S_j is released
      const uint32_t s_addr = lane_addr + TM_S;
      if (!mbar_wait_warp(&sh->s_full, (uint32_t)(j & 1), limit_ns)) { ok = false; break; }
      tc_fence_after();
      float p[64];
      {
        uint32_t sr0[32], sr1[32];  // both chunks of this half, one wait
        tmem_ld32(s_addr + (2 * half) * 32, sr0);
        tmem_ld32(s_addr + (2 * half + 1) * 32, sr1);
        tmem_ld_wait();
        exp_chunk(sr0, scale_log2, l2, (2 * half) * 32, valid, p);
        exp_chunk(sr1, scale_log2, l2, (2 * half + 1) * 32, valid, p + 32);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->s_read);
      // dS = P (dP - D) over this half's own dP columns, read first
      if (!mbar_wait_warp(&sh->dp_full, (uint32_t)(j & 1), limit_ns)) { ok = false; break; }
      tc_fence_after();
      {
        uint32_t pr[2][32];
        tmem_ld32(lane_addr + TM_DP + (2 * half) * 32, pr[0]);
        tmem_ld32(lane_addr + TM_DP + (2 * half + 1) * 32, pr[1]);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          uint32_t dsp[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            dsp[i] = pack_bf16x2(p[cc * 32 + 2 * i] * (__uint_as_float(pr[cc][2 * i]) - Dr),
                                 p[cc * 32 + 2 * i + 1] * (__uint_as_float(pr[cc][2 * i + 1]) - Dr));
          tmem_st16(lane_addr + TM_DP + 64 * half + 16 * cc, dsp);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->ds_full);
    }
    if (ok && n >= 1) ok = mbar_wait_warp(&sh->mm_done, (uint32_t)((n - 1) & 1), limit_ns);
    if (!ok) {
      bwd_timeout(sh, status);
    } else {
      tc_fence_after();
      const int row = qt * 128 + r;
      float* dst = dq + (((size_t)b * N + row) * heads + h) * D;
#pragma unroll
      for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
        uint32_t g[32];
        if (n >= 1) {
          tmem_ld32(lane_addr + TM_DQ + c * 32, g);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) g[i] = 0u;
        }
        if (row < N) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            float4 val = make_float4(__uint_as_float(g[i]) * scale, __uint_as_float(g[i + 1]) * scale,
                                     __uint_as_float(g[i + 2]) * scale, __uint_as_float(g[i + 3]) * scale);
            float4* p4 = reinterpret_cast<float4*>(dst + c * 32 + i);
            if (accumulate) {  // the linear branch's part is already there
              const float4 prev = *p4;
              val.x += prev.x;
              val.y += prev.y;
              val.z += prev.z;
              val.w += prev.w;
            }
            *p4 = val;
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ dK, dV
template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const int32_t* __restrict__ t_row_ptr, const int32_t* __restrict__ t_col_idx,
                    const float* __restrict__ lse2, const float* __restrict__ dvec, float* __restrict__ dk,
                    float* __restrict__ dv, int N, int heads, int nb, int npad, int mask_per_bh, float scale,
                    float scale_log2, uint32_t* status, uint64_t limit_ns) {
  using C = BwdCfg<D>;
  // S^T [0,128), dP^T [128,256), dV [256,256+D), dK [384,384+D).  Each row warp
  // owns 32 query columns of each query half (columns [64 h + 32 e, + 32) of S^T
  // and dP^T, e = (warp - 2) / 4) and writes P^T and dS^T of those queries as
  // bf16 pairs over the S^T columns it has read: P^T at [64 h + 32 e, + 16),
  // dS^T at [64 h + 32 e + 16, + 16).
  constexpr uint32_t TM_S = 0, TM_DP = 128, TM_DV = 256, TM_DK = 384;
  extern __shared__ uint8_t bwd_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(bwd_smem_raw) + 1023) & ~uintptr_t(1023));
  BwdShared* sh = reinterpret_cast<BwdShared*>(smem + C::OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = blockIdx.x % nb, bh = blockIdx.x / nb, b = bh / heads, h = bh % heads;
  const int mrow = (mask_per_bh ? bh : h) * nb + kt;
  const int mask_rows = (mask_per_bh ? (int)(gridDim.x / nb) : heads) * nb;
  const int c0 = t_row_ptr[mrow];
  const int n =
      debug_row_ok(t_row_ptr, t_col_idx, mrow, mask_rows, nb, true, status) ? t_row_ptr[mrow + 1] - c0 : 0;

  if (threadIdx.x == 0) {
    mbar_init(&sh->fixed_full, 1);
    mbar_init(&sh->ring_full[0], 1);
    mbar_init(&sh->ring_full[1], 1);
    mbar_init(&sh->s_full, 1);
    mbar_init(&sh->dp_full, 1);
    mbar_init(&sh->dp_read, 8);
    mbar_init(&sh->ds_h[0], 8);
    mbar_init(&sh->ds_h[1], 8);
    mbar_init(&sh->grads_done, 1);
    mbar_init(&sh->mm_done, 1);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t k_s = sbase + C::OFF_FIX, v_s = k_s + C::TILE;

  if (warp == 0) {
    if (lane == 0) {
      bool ok = true;
      int loads = 0;
      auto load_q = [&](int j) {
        const int s = j & 1, qi = t_col_idx[c0 + j];
        uint8_t* dst = smem + C::OFF_RING + s * 2 * C::TILE;
        float* vec = reinterpret_cast<float*>(smem + C::OFF_VEC + s * C::VEC);
        mbar_arrive_expect_tx(&sh->ring_full[s], 2 * C::TILE + C::VEC);
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch) {
          tma_load_3d(dst + ch * 16384, &tm_q, &sh->ring_full[s], h * D + ch * 64, qi * 128, b);
          tma_load_3d(dst + C::TILE + ch * 16384, &tm_do, &sh->ring_full[s], h * D + ch * 64, qi * 128, b);
        }
        bulk_load(vec, lse2 + (size_t)bh * npad + qi * 128, 512, &sh->ring_full[s]);
        bulk_load(vec + 128, dvec + (size_t)bh * npad + qi * 128, 512, &sh->ring_full[s]);
        ++loads;
      };
      mbar_arrive_expect_tx(&sh->fixed_full, 2 * C::TILE);
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch) {
        tma_load_3d(smem + C::OFF_FIX + ch * 16384, &tm_k, &sh->fixed_full, h * D + ch * 64, kt * 128, b);
        tma_load_3d(smem + C::OFF_FIX + C::TILE + ch * 16384, &tm_v, &sh->fixed_full, h * D + ch * 64, kt * 128, b);
      }
      for (int j = 0; j < n && j < 2; ++j) load_q(j);
      ok = mbar_wait(&sh->fixed_full, 0, limit_ns);
      if (ok && n >= 1) {
        ok = mbar_wait(&sh->ring_full[0], 0, limit_ns);
        if (ok) {
          tc_fence_after();
          const uint32_t qs = sbase + C::OFF_RING;
          mma_xyt<D>(tmem + TM_S, k_s, qs);
          mma_commit(&sh->s_full);
          mma_xyt<D>(tmem + TM_DP, v_s, qs + C::TILE);
          mma_commit(&sh->dp_full);
        }
      }
      // Per tile: dP^T_{j+1} as soon as the row warps hold dP^T_j in registers;
      // the gradient products of query half 0 while they form half 1; then those
      // of half 1 and S^T_{j+1}, which overwrites the P^T / dS^T they read (the
      // tensor cores run them in issue order).
      for (int j = 0; ok && j < n; ++j) {
        const uint32_t qs = sbase + C::OFF_RING + (j & 1) * 2 * C::TILE;
        const uint32_t qn = sbase + C::OFF_RING + ((j + 1) & 1) * 2 * C::TILE;
        if (j + 1 < n) {
          if (sh->abort_flag || !mbar_wait(&sh->dp_read, (uint32_t)(j & 1), limit_ns) ||
              !mbar_wait(&sh->ring_full[(j + 1) & 1], (uint32_t)(((j + 1) >> 1) & 1), limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_xyt<D>(tmem + TM_DP, v_s, qn + C::TILE);
          mma_commit(&sh->dp_full);
        }
        for (int ph = 0; ph < 2; ++ph) {
          if (sh->abort_flag || !mbar_wait(&sh->ds_h[ph], (uint32_t)(j & 1), limit_ns)) { ok = false; break; }
          tc_fence_after();
          const bool acc = j > 0 || ph > 0;
          mma_grad_half<D>(tmem + TM_DV, tmem + TM_S + 64 * ph, qs + C::TILE + ph * 8192, acc);  // dV += P^T dO
          mma_grad_half<D>(tmem + TM_DK, tmem + TM_S + 64 * ph + 16, qs + ph * 8192, acc);       // dK += dS^T Q
        }
        if (!ok) break;
        mma_commit(j + 1 < n ? &sh->mm_done : &sh->grads_done);
        if (j + 1 < n) {
          mma_xyt<D>(tmem + TM_S, k_s, qn);
          mma_commit(&sh->s_full);
        }
        if (j + 2 < n) {
          // the stage of tile j is free once its gradient products have read it
          if (!mbar_wait(&sh->mm_done, (uint32_t)(j & 1), limit_ns)) { ok = false; break; }
          load_q(j + 2);
        }
      }
      if (!ok) {
        bwd_timeout(sh, status);
        mma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kBwdDrainNs);
      }
      mbar_wait(&sh->fixed_full, 0, kBwdDrainNs);
      for (int i = (loads > 2 ? loads - 2 : 0); i < loads; ++i)
        mbar_wait(&sh->ring_full[i & 1], (uint32_t)((i >> 1) & 1), kBwdDrainNs);
    }
  } else if (warp >= 2) {
    // ---------------------------------------------------------- one thread per key row
    // and 32 query columns of each query half: [64 ph + 32 half, + 32)
    const int quarter = warp & 3, r = quarter * 32 + lane, half = (warp - 2) >> 2;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int s = j & 1;
      if (!mbar_wait_warp(&sh->s_full, (uint32_t)(j & 1), limit_ns) ||
          !mbar_wait_warp(&sh->dp_full, (uint32_t)(j & 1), limit_ns)) {
        ok = false;
        break;
      }
      // the row vectors of this query tile landed with its tiles (ring_full of stage s)
      if (!mbar_wait_warp(&sh->ring_full[s], (uint32_t)((j >> 1) & 1), limit_ns)) { ok = false; break; }
      tc_fence_after();
      const float* l2v = reinterpret_cast<const float*>(smem + C::OFF_VEC + s * C::VEC);
      const float* dvv = l2v + 128;
      uint32_t sr2[2][32], pr2[2][32];  // this thread's chunks of S^T and dP^T, one wait
#pragma unroll
      for (int ph = 0; ph < 2; ++ph) {
        tmem_ld32(lane_addr + TM_S + 64 * ph + 32 * half, sr2[ph]);
        tmem_ld32(lane_addr + TM_DP + 64 * ph + 32 * half, pr2[ph]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->dp_read);  // dP^T_j is in registers: its columns are free
#pragma unroll
      for (int ph = 0; ph < 2; ++ph) {
        const uint32_t(&sr)[32] = sr2[ph];
        const uint32_t(&pr)[32] = pr2[ph];
        uint32_t pp[16], dsp[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int q0 = 64 * ph + 32 * half + 2 * i;
          const uint64_t x = f32x2_fma(f32x2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])),
                                       f32x2_pack(scale_log2, scale_log2), f32x2_pack(-l2v[q0], -l2v[q0 + 1]));
          float p0, p1;
          if ((i & 3) == 3) {
            exp2_fma_x2(x, p0, p1);  // one pair in four on the FMA pipe
          } else {
            float x0, x1;
            f32x2_unpack(x, x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          pp[i] = pack_bf16x2(p0, p1);
          dsp[i] = pack_bf16x2(p0 * (__uint_as_float(pr[2 * i]) - dvv[q0]),
                               p1 * (__uint_as_float(pr[2 * i + 1]) - dvv[q0 + 1]));
        }
        tmem_st16(lane_addr + TM_S + 64 * ph + 32 * half, pp);
        tmem_st16(lane_addr + TM_S + 64 * ph + 32 * half + 16, dsp);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->ds_h[ph]);
      }
    }
    if (ok && n >= 1) ok = mbar_wait_warp(&sh->grads_done, 0, limit_ns);
    if (!ok) {
      bwd_timeout(sh, status);
    } else {
      tc_fence_after();
      const int row = kt * 128 + r;
      const size_t off = (((size_t)b * N + row) * heads + h) * D;
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float* dst = (part == 0 ? dv : dk) + off;
        const float mul = part == 0 ? 1.f : scale;
#pragma unroll
        for (int c = half * (D / 64); c < (half + 1) * (D / 64); ++c) {
          uint32_t g[32];
          if (n >= 1) {
            tmem_ld32(lane_addr + (part == 0 ? TM_DV : TM_DK) + c * 32, g);
            tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) g[i] = 0u;
          }
          if (row < N) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              *reinterpret_cast<float4*>(dst + c * 32 + i) =
                  make_float4(__uint_as_float(g[i]) * mul, __uint_as_float(g[i + 1]) * mul,
                              __uint_as_float(g[i + 2]) * mul, __uint_as_float(g[i + 3]) * mul);
          }
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D>
cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t s) {
  using C = BwdCfg<D>;
  const long long rows = (long long)a.B * a.heads * a.npad;
  cudaError_t e = cudaSuccess;
  if (!a.full) {  // with the linear branch the row kernel has written lse2 and D
    bwd_prep_kernel<D><<<(unsigned)((rows + 255) / 256), 256, 0, s>>>(a.o, a.dout, a.lse, a.B, a.N, a.heads, a.npad,
                                                                     a.lse2, a.dvec);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int grid = a.B * a.heads * a.nb;
  e = cudaFuncSetAttribute(bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::DQ_SMEM);
  if (e != cudaSuccess) return e;
  bwd_dq_kernel<D><<<grid, kBwdThreads, C::DQ_SMEM, s>>>(*a.tm_q, *a.tm_k, *a.tm_v, *a.tm_do, a.row_ptr, a.col_idx,
                                                      a.lse2, a.dvec, a.dq, a.N, a.heads, a.nb, a.npad,
                                                      a.mask_per_bh, a.scale, a.scale_log2, a.status,
                                                      a.wait_limit_ns, a.full);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bwd_dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  bwd_dkdv_kernel<D><<<grid, kBwdThreads, C::SMEM, s>>>(*a.tm_q, *a.tm_k, *a.tm_v, *a.tm_do, a.t_row_ptr,
                                                        a.t_col_idx, a.lse2, a.dvec, a.dk, a.dv, a.N, a.heads, a.nb,
                                                        a.npad, a.mask_per_bh, a.scale, a.scale_log2, a.status,
                                                        a.wait_limit_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_backward(const BwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_bwd_t<64>(a, s) : launch_bwd_t<128>(a, s);
}

}  // namespace salad
