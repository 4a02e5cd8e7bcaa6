// Backward pass of the linear branch, its projection and the gate, on the
// tensor cores (the sparse branch's gradients are in bwd.cu).  SALAD summary
// section 2.1 defines the branch: per (b, h), with the state S, z of linear.cu,
// a_i = relu(q_i), den_i = a_i.z + eps, o_i = a_i S / den_i, out_i gets g o_i W.
// With T = S W (the projected state of the forward), G_i = dL/dout_i and
//   P1_i = a_i T,  P2_i = G_i T^T                          (row products)
//   yg_i = G_i.P1_i / den_i  (= G_i.(o_i W)),  s_i = g / den_i,  dden_i = -g yg_i / den_i
// the gradients are
//   dgate = sum_i yg_i
//   dq_i  = [q_i > 0] (s_i P2_i + dden_i z)       (the sparse branch's part is added later)
//   M     = sum_i a_i^T (s_i G_i)                 (d x d)
//   dS    = M W^T,  dz = sum_i dden_i a_i,  dW = sum over (b, h) of S^T M
//   dk_j += [k_j > 0] (v_j dS^T + dz),  dv_j += relu(k_j) dS
// and the sparse branch's D_i = G_i.out_i - g yg_i (its output is out_i - g o_i W).
// These follow from dy_i = g G_i, do_i = dy_i W^T, du_i = do_i / den_i:
// do_i.o_i = g yg_i, S du_i = s_i T G_i, sum_i a_i du_i^T = M W^T and
// sum_i o_i^T dy_i = S^T M.
//
//   lin_rows_kernel        grid (splits, B*Hh): each CTA streams 128-row tiles of
//                          one (b, h) through a two-stage TMA ring; one thread
//                          issues P1 = A [T_hi; T_lo] and P2 = G [T_hi; T_lo]^T
//                          into tensor memory, four warps turn each row into dq,
//                          D_i, lse2, dden_i and the row of X = s_i G_i (bf16 hi +
//                          lo), and M += A^T X_hi + A^T X_lo accumulates in tensor
//                          memory across the CTA's tiles.  Per split: M, dz, dgate.
//   lin_state_grad_kernel  the splits in order: dS = M W^T as bf16 hi + lo operand
//                          halves, dz, dgate, and S^T M over 16 rows of S and M
//   lin_dw_kernel          dW: those partials in (b, h) then row-block order
//   lin_keys_kernel        grid (splits, B*Hh): per 128 key rows, V [dS_hi; dS_lo]^T
//                          and relu(K) [dS_hi; dS_lo] in double-buffered tensor
//                          memory, added to the sparse branch's dk and dv.
// Every sum runs in a fixed order, so the gradients do not vary run to run.
#include "internal.h"
#include "ptx.cuh"

namespace salad {
namespace {

constexpr uint64_t kDrainNs = 1000000000ull;
constexpr float kLog2eL = 1.4426950408889634f;

// Shared layout of both streaming kernels: an operand of d x d bf16 hi + lo
// halves (T or dS: 2d/64 chunks of [d rows x 64 columns], 128-byte swizzle),
// then two stages of two 128-row tiles.
template <int D>
struct LinBwdCfg {
  static constexpr int BOX = 128 * 128;                 // [128 rows x 64 columns] bf16
  static constexpr int TILE = (D / 64) * BOX;           // a 128 x D tile
  static constexpr int OP_CH = D * 128;                 // [D rows x 64 columns] bf16
  static constexpr int OP_BYTES = 2 * (D / 64) * OP_CH;  // hi chunks, then lo chunks
  static constexpr int STAGES = 2;
  static constexpr int OFF_STAGE = OP_BYTES;            // stage s: first tile, then second tile
  static constexpr int OFF_XLO = OFF_STAGE + STAGES * 2 * TILE;  // rows kernel only
  static constexpr int ROWS_OFF_BAR = OFF_XLO + TILE;
  static constexpr int KEYS_OFF_BAR = OFF_XLO;
  static constexpr uint32_t IDESC_NN = idesc_bf16(128, D, false, false);  // both K-major
  static constexpr uint32_t IDESC_NT = idesc_bf16(128, D, false, true);   // B MN-major
  static constexpr uint32_t IDESC_TT = idesc_bf16(128, D, true, true);    // A and B MN-major
  static constexpr uint32_t TMEM_COLS = D == 128 ? 512 : 256;
  // CTAs one SM holds: shared memory allows one at d = 128, two at d = 64.
  static constexpr int CTAS_PER_SM = D == 128 ? 1 : 2;
};

struct RowShared {
  uint64_t full[2], empty[2];
  uint64_t op_full, relu, p_full, p_free, x_full, x_free, dd_bar, m_done, drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  float zs[128];
  float dden[2][128];
  float red[4];
};

struct KeyShared {
  uint64_t full[2], empty[2];
  uint64_t op_full, relu, acc_full[2], acc_free[2], drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  float dzs[128];
};

template <int D>
constexpr int rows_smem() { return LinBwdCfg<D>::ROWS_OFF_BAR + (int)sizeof(RowShared) + 1024; }
template <int D>
constexpr int keys_smem() { return LinBwdCfg<D>::KEYS_OFF_BAR + (int)sizeof(KeyShared) + 1024; }
static_assert(rows_smem<128>() <= 232448, "rows kernel shared memory");
static_assert(keys_smem<128>() <= 232448, "keys kernel shared memory");

template <typename Sh>
__device__ __forceinline__ void record_timeout(Sh* sh, uint32_t* status) {
  sh->abort_flag = 1;
  atomicOr(status, kStatusTimeout);
}

// Bounded wait taken by a whole warp, false (in every lane) once the CTA is
// aborting or the wait timed out, so the warp never diverges around it.
template <typename Sh>
__device__ __forceinline__ bool warp_wait(Sh* sh, uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (__any_sync(0xffffffffu, sh->abort_flag != 0)) return false;
  return mbar_wait_warp(bar, parity, limit_ns);
}

__device__ __forceinline__ uint32_t relu2(uint32_t v) {
  const uint32_t neg = ((v >> 15) & 0x00010001u) * 0xFFFFu;  // 0xFFFF in each negative half
  return v & ~neg;
}

// Row r of a 128-row tile (D / 64 boxes): ReLU in place; returns sum_c relu(x_c) z_c.
template <int D>
__device__ __forceinline__ float relu_row(uint32_t tile, int r, const float* z) {
  float d0 = 0.f, d1 = 0.f;
#pragma unroll
  for (int ch = 0; ch < D / 64; ++ch)
#pragma unroll
    for (int p = 0; p < 8; ++p) {
      const uint32_t addr = tile + ch * LinBwdCfg<D>::BOX + sw128_offset((uint32_t)r, (uint32_t)p);
      uint32_t x[4];
      ld_shared_v4(addr, x[0], x[1], x[2], x[3]);
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] = relu2(x[i]);
      st_shared_v4(addr, x[0], x[1], x[2], x[3]);
      if (z != nullptr) {
        const int c = ch * 64 + p * 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          d0 = fmaf(bf16_lo_to_f32(x[i]), z[c + 2 * i], d0);
          d1 = fmaf(bf16_hi_to_f32(x[i]), z[c + 2 * i + 1], d1);
        }
      }
    }
  return d0 + d1;
}

// ReLU in place on columns [half D / 2, half D / 2 + D / 2) of row r of a
// 128-row tile.
template <int D>
__device__ __forceinline__ void relu_half_row(uint32_t tile, int r, int half) {
#pragma unroll
  for (int pp = 0; pp < D / 16; ++pp) {
    const int piece = half * (D / 16) + pp;  // 16-byte piece of the row: chunk piece / 8
    const uint32_t addr = tile + (piece / 8) * LinBwdCfg<D>::BOX + sw128_offset((uint32_t)r, (uint32_t)(piece % 8));
    uint32_t x[4];
    ld_shared_v4(addr, x[0], x[1], x[2], x[3]);
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = relu2(x[i]);
    st_shared_v4(addr, x[0], x[1], x[2], x[3]);
  }
}

// The 32 bf16 of columns 32 cc ... 32 cc + 31 of row r of a tile, as 16 pairs.
template <int D>
__device__ __forceinline__ void tile_cols32(uint32_t tile, int r, int cc, uint32_t (&x)[16]) {
#pragma unroll
  for (int j = 0; j < 4; ++j)
    ld_shared_v4(tile + (cc / 2) * LinBwdCfg<D>::BOX + sw128_offset((uint32_t)r, (uint32_t)((cc % 2) * 4 + j)),
                 x[4 * j], x[4 * j + 1], x[4 * j + 2], x[4 * j + 3]);
}

// ------------------------------------------------------------------ rows
template <int D>
__global__ void __launch_bounds__(192, 1)
    lin_rows_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_t, const uint16_t* __restrict__ out,
                    const float* __restrict__ lse, const float* __restrict__ gate, const float* __restrict__ zvec,
                    int N, int heads, int npad, int tiles_per_split, float eps, float* __restrict__ dq,
                    float* __restrict__ lse2, float* __restrict__ dvec, float* __restrict__ m_part,
                    float* __restrict__ dz_part, float* __restrict__ dg_part, uint32_t* status, uint64_t limit_ns) {
  using C = LinBwdCfg<D>;
  const int split = blockIdx.x, bh = blockIdx.y, BH = gridDim.y;
  const int b = bh / heads, h = bh % heads;
  const int ntiles = (N + 127) / 128;
  const int t_begin = split * tiles_per_split;
  const int n_tiles = min(ntiles, t_begin + tiles_per_split) - t_begin;  // >= 1 by construction

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  RowShared* sh = reinterpret_cast<RowShared*>(smem + C::ROWS_OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1 + 4);  // the MMA commit and the four row warps
    }
    mbar_init(&sh->op_full, 1);
    mbar_init(&sh->relu, 4);
    mbar_init(&sh->p_full, 1);
    mbar_init(&sh->p_free, 4);
    mbar_init(&sh->x_full, 4);
    mbar_init(&sh->x_free, 1);
    mbar_init(&sh->dd_bar, 128);
    mbar_init(&sh->m_done, 1);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tm_q);
    tma_prefetch_map(&tm_do);
    tma_prefetch_map(&tm_t);
  }
  if (threadIdx.x < D) sh->zs[threadIdx.x] = zvec[(size_t)bh * D + threadIdx.x];
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  constexpr uint32_t TM_P1 = 0, TM_P2 = D, TM_M = 2 * D;
  const uint32_t op = sbase;  // T hi | lo

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&sh->op_full, C::OP_BYTES);
#pragma unroll
      for (int ch = 0; ch < 2 * D / 64; ++ch) tma_load_3d(smem + ch * C::OP_CH, &tm_t, &sh->op_full, ch * 64, 0, bh);
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int s = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        if (sh->abort_flag || !mbar_wait(&sh->empty[s], ph ^ 1, limit_ns)) {
          record_timeout(sh, status);
          break;
        }
        uint8_t* at = smem + C::OFF_STAGE + s * 2 * C::TILE;
        mbar_arrive_expect_tx(&sh->full[s], 2 * C::TILE);
        const int row0 = (t_begin + it) * 128;
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
          tma_load_3d(at + ch * C::BOX, &tm_q, &sh->full[s], h * D + ch * 64, row0, b);
          tma_load_3d(at + C::TILE + ch * C::BOX, &tm_do, &sh->full[s], h * D + ch * 64, row0, b);
        }
        issued = it + 1;
      }
      if (sh->abort_flag) {
        // let every copy this thread started land before the CTA can exit
        mbar_wait(&sh->op_full, 0, kDrainNs);
        for (int it = (issued > 2 ? issued - 2 : 0); it < issued; ++it)
          mbar_wait(&sh->full[it & 1], (it >> 1) & 1, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sh->op_full, 0, limit_ns);
      if (!ok) record_timeout(sh, status);
      for (int it = 0; it < n_tiles && ok; ++it) {
        const int s = it & 1;
        if (sh->abort_flag || !mbar_wait(&sh->relu, it & 1, limit_ns) ||
            (it > 0 && !mbar_wait(&sh->p_free, (it - 1) & 1, limit_ns))) {
          record_timeout(sh, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t at = sbase + C::OFF_STAGE + s * 2 * C::TILE, gt = at + C::TILE;
        // P1 = A T: B rows are f (N), K = c runs along them (K-major)
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sw128_desc(at + (kk / 4) * C::BOX + (kk % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(op + (hl * (D / 64) + kk / 4) * C::OP_CH + (kk % 4) * 32, 16, 1024);
            mma_bf16_ss(tmem + TM_P1, a, bd, C::IDESC_NN, (hl | kk) ? 1u : 0u);
          }
        // P2 = G T^T: the same rows f are now K, c runs along them (MN-major)
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sw128_desc(gt + (kk / 4) * C::BOX + (kk % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(op + hl * (D / 64) * C::OP_CH + kk * 2048, C::OP_CH, 1024);
            mma_bf16_ss(tmem + TM_P2, a, bd, C::IDESC_NT, (hl | kk) ? 1u : 0u);
          }
        mma_commit(&sh->p_full);
        if (sh->abort_flag || !mbar_wait(&sh->x_full, it & 1, limit_ns)) {
          record_timeout(sh, status);
          ok = false;
          break;
        }
        tc_fence_after();
        // M += A^T X: K = the 128 rows of the tile, A^T and X both MN-major.
        // At d = 64 the second 64-wide half of A^T reads the G tile and lands in
        // accumulator rows 64..127, which are never read.
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t a = sw128_desc(at + kk * 2048, C::BOX, 1024);
            const uint64_t bd = sw128_desc((hl ? sbase + C::OFF_XLO : gt) + kk * 2048, C::BOX, 1024);
            mma_bf16_ss(tmem + TM_M, a, bd, C::IDESC_TT, (it | hl | kk) ? 1u : 0u);
          }
        mma_commit(&sh->empty[s]);
        mma_commit(&sh->x_free);
      }
      if (ok) {
        mma_commit(&sh->m_done);
      } else {
        mma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kDrainNs);
      }
    }
  } else {
    // ---------------- row warps 2..5: thread (quarter, lane) owns row 32 quarter + lane
    const int t = threadIdx.x - 64;
    const int quarter = warp & 3, r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    const float g = gate[bh];
    // dz: thread t sums the column pair (2 pr, 2 pr + 1) over row group rg of every tile
    constexpr int PAIRS = D / 2, RG = 128 / PAIRS, RPG = 128 / RG;
    const int pr = t % PAIRS, rg = t / PAIRS;
    float dg_acc = 0.f, dz_acc0 = 0.f, dz_acc1 = 0.f;
    bool ok = true;
    for (int it = 0; it < n_tiles; ++it) {
      const int s = it & 1;
      const uint32_t ph = (it >> 1) & 1;
      const uint32_t at = sbase + C::OFF_STAGE + s * 2 * C::TILE, gt = at + C::TILE, xlo = sbase + C::OFF_XLO;
      const int row = (t_begin + it) * 128 + r;
      // the row of the output, for D_i: its loads are in flight during the waits below
      const bool live = row < N;
      uint4 ov[D / 8];
      {
        const uint4* orow = reinterpret_cast<const uint4*>(out + (((size_t)b * N + (live ? row : 0)) * heads + h) * D);
#pragma unroll
        for (int j = 0; j < D / 8; ++j) ov[j] = live ? __ldg(orow + j) : make_uint4(0, 0, 0, 0);
      }
      // 1. ReLU of the row of q in place, den
      if (!warp_wait(sh, &sh->full[s], ph, limit_ns)) {
        ok = false;
        break;
      }
      const float den = relu_row<D>(at, r, sh->zs) + eps;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->relu);
      // 2. yg and G.out from P1
      if (!warp_wait(sh, &sh->p_full, it & 1, limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float yg0 = 0.f, yg1 = 0.f, go0 = 0.f, go1 = 0.f;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t p1[32], gx[16];
        tmem_ld32(lane_base + TM_P1 + cc * 32, p1);
        tile_cols32<D>(gt, r, cc, gx);
        tmem_ld_wait();
        const uint32_t* ow = reinterpret_cast<const uint32_t*>(&ov[cc * 4]);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float ga = bf16_lo_to_f32(gx[i]), gb = bf16_hi_to_f32(gx[i]);
          yg0 = fmaf(ga, __uint_as_float(p1[2 * i]), yg0);
          yg1 = fmaf(gb, __uint_as_float(p1[2 * i + 1]), yg1);
          go0 = fmaf(ga, bf16_lo_to_f32(ow[i]), go0);
          go1 = fmaf(gb, bf16_hi_to_f32(ow[i]), go1);
        }
      }
      const float yg = (yg0 + yg1) / den;
      const float dden = -g * yg / den;
      const float sg = g / den;
      // 3. the row of X = s_i G_i as bf16 hi (over G) and lo (its own buffer)
      if (it > 0 && !warp_wait(sh, &sh->x_free, (it - 1) & 1, limit_ns)) {
        ok = false;
        break;
      }
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch)
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const uint32_t off = ch * C::BOX + sw128_offset((uint32_t)r, (uint32_t)p);
          uint32_t x[4], hi[4], lo[4];
          ld_shared_v4(gt + off, x[0], x[1], x[2], x[3]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float v0 = sg * bf16_lo_to_f32(x[i]), v1 = sg * bf16_hi_to_f32(x[i]);
            hi[i] = pack_bf16x2(v0, v1);
            lo[i] = pack_bf16x2(v0 - bf16_lo_to_f32(hi[i]), v1 - bf16_hi_to_f32(hi[i]));
          }
          st_shared_v4(gt + off, hi[0], hi[1], hi[2], hi[3]);
          st_shared_v4(xlo + off, lo[0], lo[1], lo[2], lo[3]);
        }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->x_full);
      // 4. dq = [q > 0] (s_i P2 + dden z)
      float* dqrow = dq + (((size_t)b * N + (live ? row : 0)) * heads + h) * D;
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t p2[32], ax[16];
        tmem_ld32(lane_base + TM_P2 + cc * 32, p2);
        tile_cols32<D>(at, r, cc, ax);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c = cc * 32 + 2 * i;
          v[2 * i] = (ax[i] & 0xFFFFu) ? fmaf(sg, __uint_as_float(p2[2 * i]), dden * sh->zs[c]) : 0.f;
          v[2 * i + 1] = (ax[i] >> 16) ? fmaf(sg, __uint_as_float(p2[2 * i + 1]), dden * sh->zs[c + 1]) : 0.f;
        }
        if (live) {
#pragma unroll
          for (int j = 0; j < 8; ++j)
            reinterpret_cast<float4*>(dqrow + cc * 32)[j] =
                make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->p_free);
      // 5. per-row outputs for the sparse backward, dgate, and dz over the tile's rows
      if (live) {
        dvec[(size_t)bh * npad + row] = go0 + go1 - g * yg;
        lse2[(size_t)bh * npad + row] = lse[(size_t)bh * N + row] * kLog2eL;
      } else if (row < npad) {
        dvec[(size_t)bh * npad + row] = 0.f;  // pad rows: no probability mass
        lse2[(size_t)bh * npad + row] = INFINITY;
      }
      dg_acc += yg;
      sh->dden[it & 1][r] = dden;
      mbar_arrive(&sh->dd_bar);
      if (!warp_wait(sh, &sh->dd_bar, it & 1, limit_ns)) {
        ok = false;
        break;
      }
      {
        // column pair (2 pr, 2 pr + 1): chunk pr / 32, 16-byte piece (pr % 32) / 4, word pr % 4
        const uint32_t col = at + (pr / 32) * C::BOX + (uint32_t)(pr % 4) * 4;
        const uint32_t piece = (uint32_t)((pr % 32) / 4);
        float z0 = 0.f, z1 = 0.f;
#pragma unroll 8
        for (int i = rg * RPG; i < (rg + 1) * RPG; ++i) {
          uint32_t a2;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(a2) : "r"(col + sw128_offset((uint32_t)i, piece)));
          const float dd = sh->dden[it & 1][i];
          z0 = fmaf(bf16_lo_to_f32(a2), dd, z0);
          z1 = fmaf(bf16_hi_to_f32(a2), dd, z1);
        }
        dz_acc0 += z0;
        dz_acc1 += z1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->empty[s]);
    }
    if (!ok) record_timeout(sh, status);
    ok = __all_sync(0xffffffffu, ok);
    // dgate: fixed-order sum over the 128 threads (shuffle tree, then the four warps in order)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dg_acc += __shfl_xor_sync(0xffffffffu, dg_acc, o);
    const size_t part = (size_t)split * BH + bh;
    if (lane == 0) sh->red[warp - 2] = dg_acc;
    if (ok) {
      dz_part[(part * RG + rg) * D + 2 * pr] = dz_acc0;
      dz_part[(part * RG + rg) * D + 2 * pr + 1] = dz_acc1;
      if (warp_wait(sh, &sh->m_done, 0, limit_ns)) {
        tc_fence_after();
        if (quarter * 32 < D) {
          float* mrow = m_part + (part * D + quarter * 32 + lane) * D;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t m[32];
            tmem_ld32(lane_base + TM_M + cc * 32, m);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 8; ++j)
              reinterpret_cast<float4*>(mrow + cc * 32)[j] =
                  make_float4(__uint_as_float(m[4 * j]), __uint_as_float(m[4 * j + 1]),
                              __uint_as_float(m[4 * j + 2]), __uint_as_float(m[4 * j + 3]));
          }
        }
      } else {
        record_timeout(sh, status);
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  // dgate partial: the four row warps' sums in order
  if (threadIdx.x == 64 && !sh->abort_flag)
    dg_part[(size_t)split * BH + bh] = (sh->red[0] + sh->red[1]) + (sh->red[2] + sh->red[3]);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ keys
template <int D>
__global__ void __launch_bounds__(320, 1)
    lin_keys_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CUtensorMap tm_ds, const float* __restrict__ dz, int N, int heads,
                    int tiles_per_split, float* __restrict__ dk, float* __restrict__ dv, uint32_t* status,
                    uint64_t limit_ns) {
  using C = LinBwdCfg<D>;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / heads, h = bh % heads;
  const int ntiles = (N + 127) / 128;
  const int t_begin = split * tiles_per_split;
  const int n_tiles = min(ntiles, t_begin + tiles_per_split) - t_begin;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  KeyShared* sh = reinterpret_cast<KeyShared*>(smem + C::KEYS_OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1 + 8);  // the MMA commit and the eight row warps
      mbar_init(&sh->acc_full[s], 1);
      mbar_init(&sh->acc_free[s], 8);
    }
    mbar_init(&sh->op_full, 1);
    mbar_init(&sh->relu, 8);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
    tma_prefetch_map(&tm_ds);
  }
  if (threadIdx.x < D) sh->dzs[threadIdx.x] = dz[(size_t)bh * D + threadIdx.x];
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
  const uint32_t op = sbase;  // dS hi | lo, rows c

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(&sh->op_full, C::OP_BYTES);
#pragma unroll
      for (int ch = 0; ch < 2 * D / 64; ++ch) tma_load_3d(smem + ch * C::OP_CH, &tm_ds, &sh->op_full, ch * 64, 0, bh);
      int issued = 0;
      for (int it = 0; it < n_tiles; ++it) {
        const int s = it & 1;
        const uint32_t ph = (it >> 1) & 1;
        if (sh->abort_flag || !mbar_wait(&sh->empty[s], ph ^ 1, limit_ns)) {
          record_timeout(sh, status);
          break;
        }
        uint8_t* kt = smem + C::OFF_STAGE + s * 2 * C::TILE;
        mbar_arrive_expect_tx(&sh->full[s], 2 * C::TILE);
        const int row0 = (t_begin + it) * 128;
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
          tma_load_3d(kt + ch * C::BOX, &tm_k, &sh->full[s], h * D + ch * 64, row0, b);
          tma_load_3d(kt + C::TILE + ch * C::BOX, &tm_v, &sh->full[s], h * D + ch * 64, row0, b);
        }
        issued = it + 1;
      }
      if (sh->abort_flag) {
        mbar_wait(&sh->op_full, 0, kDrainNs);
        for (int it = (issued > 2 ? issued - 2 : 0); it < issued; ++it)
          mbar_wait(&sh->full[it & 1], (it >> 1) & 1, kDrainNs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(&sh->op_full, 0, limit_ns);
      if (!ok) record_timeout(sh, status);
      for (int it = 0; it < n_tiles && ok; ++it) {
        const int s = it & 1, buf = it & 1;
        if (sh->abort_flag || !mbar_wait(&sh->relu, it & 1, limit_ns) ||
            !mbar_wait(&sh->acc_free[buf], ((it >> 1) & 1) ^ 1, limit_ns)) {
          record_timeout(sh, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kt = sbase + C::OFF_STAGE + s * 2 * C::TILE, vt = kt + C::TILE;
        const uint32_t acc_k = tmem + buf * 2 * D, acc_v = acc_k + D;
        // v_j dS^T: B rows are c (N), K = e runs along them (K-major)
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sw128_desc(vt + (kk / 4) * C::BOX + (kk % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(op + (hl * (D / 64) + kk / 4) * C::OP_CH + (kk % 4) * 32, 16, 1024);
            mma_bf16_ss(acc_k, a, bd, C::IDESC_NN, (hl | kk) ? 1u : 0u);
          }
        // relu(k_j) dS: the rows c are K, e runs along them (MN-major)
#pragma unroll
        for (int hl = 0; hl < 2; ++hl)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint64_t a = sw128_desc(kt + (kk / 4) * C::BOX + (kk % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(op + hl * (D / 64) * C::OP_CH + kk * 2048, C::OP_CH, 1024);
            mma_bf16_ss(acc_v, a, bd, C::IDESC_NT, (hl | kk) ? 1u : 0u);
          }
        mma_commit(&sh->acc_full[buf]);
        mma_commit(&sh->empty[s]);
      }
      if (!ok) {
        mma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kDrainNs);
      }
    }
  } else {
    // ---------------- row warps 2..9: ReLU of the next tile, then this tile's rows of
    // dk, dv; warp w takes row 32 (w % 4) + lane (its TMEM lane quarter) and the
    // column half (w - 2) / 4
    const int quarter = warp & 3, r = quarter * 32 + lane, half = (warp - 2) >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    if (n_tiles > 0) {
      if (!warp_wait(sh, &sh->full[0], 0, limit_ns)) {
        ok = false;
      } else {
        relu_half_row<D>(sbase + C::OFF_STAGE, r, half);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->relu);
      }
    }
    for (int it = 0; it < n_tiles && ok; ++it) {
      const int s = it & 1, buf = it & 1;
      if (it + 1 < n_tiles) {
        const int s1 = (it + 1) & 1;
        if (!warp_wait(sh, &sh->full[s1], ((it + 1) >> 1) & 1, limit_ns)) {
          ok = false;
          break;
        }
        relu_half_row<D>(sbase + C::OFF_STAGE + s1 * 2 * C::TILE, r, half);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->relu);
      }
      if (!warp_wait(sh, &sh->acc_full[buf], (it >> 1) & 1, limit_ns)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t kt = sbase + C::OFF_STAGE + s * 2 * C::TILE;
      const int row = (t_begin + it) * 128 + r;
      const bool live = row < N;
      const size_t off = (((size_t)b * N + (live ? row : 0)) * heads + h) * D;
#pragma unroll 1
      for (int cc = half * (D / 64); cc < (half + 1) * (D / 64); ++cc) {
        uint32_t ak[32], av[32], kx[16];
        tmem_ld32(lane_base + buf * 2 * D + cc * 32, ak);
        tmem_ld32(lane_base + buf * 2 * D + D + cc * 32, av);
        tile_cols32<D>(kt, r, cc, kx);
        float4 ok4[8], ov4[8];
        float4* dkr = reinterpret_cast<float4*>(dk + off + cc * 32);
        float4* dvr = reinterpret_cast<float4*>(dv + off + cc * 32);
        if (live) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            ok4[j] = dkr[j];
            ov4[j] = dvr[j];
          }
        }
        tmem_ld_wait();
        if (live) {
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int c = cc * 32 + 4 * j;
            const uint32_t m0 = kx[2 * j], m1 = kx[2 * j + 1];
            float4 a = ok4[j];
            a.x += (m0 & 0xFFFFu) ? __uint_as_float(ak[4 * j]) + sh->dzs[c] : 0.f;
            a.y += (m0 >> 16) ? __uint_as_float(ak[4 * j + 1]) + sh->dzs[c + 1] : 0.f;
            a.z += (m1 & 0xFFFFu) ? __uint_as_float(ak[4 * j + 2]) + sh->dzs[c + 2] : 0.f;
            a.w += (m1 >> 16) ? __uint_as_float(ak[4 * j + 3]) + sh->dzs[c + 3] : 0.f;
            dkr[j] = a;
            float4 e = ov4[j];
            e.x += __uint_as_float(av[4 * j]);
            e.y += __uint_as_float(av[4 * j + 1]);
            e.z += __uint_as_float(av[4 * j + 2]);
            e.w += __uint_as_float(av[4 * j + 3]);
            dvr[j] = e;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sh->acc_free[buf]);
        mbar_arrive(&sh->empty[s]);
      }
    }
    if (!ok) record_timeout(sh, status);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ state gradients
// grid (B*Hh, D/16), 256 threads.  CTA (bh, blk) owns rows c in [16 blk, 16 blk + 16)
// of M: it sums their split partials in split order, writes those rows of dS =
// M W^T as bf16 hi + lo halves ds_op[bh][c][e] (hi), ds_op[bh][c][D + e] (lo), the
// operand layout of lin_keys_kernel, and the partial S^T M over its 16 rows,
// dw_part[bh][blk][e][f] = sum_{c in blk} S[c][e] M[c][f].  CTA (bh, 0) also sums
// dz and dgate.
template <int D>
__global__ void __launch_bounds__(256) lin_state_grad_kernel(const float* __restrict__ m_part,
                                                             const float* __restrict__ dz_part,
                                                             const float* __restrict__ dg_part,
                                                             const float* __restrict__ S, const uint16_t* __restrict__ w,
                                                             int splits, uint16_t* __restrict__ ds_op,
                                                             float* __restrict__ dz, float* __restrict__ dgate,
                                                             float* __restrict__ dw_part) {
  extern __shared__ float sg_smem[];
  float* Ms = sg_smem;                                           // [16][D]
  float* Ss = Ms + 16 * D;                                       // [16][D]
  uint16_t* Wt = reinterpret_cast<uint16_t*>(Ss + 16 * D);       // [D][D]: Wt[f][e] = W[e][f]
  const int bh = blockIdx.x, blk = blockIdx.y, BH = gridDim.x, t = threadIdx.x;
  const int c0 = blk * 16;
  for (int x = t; x < D * D; x += 256) Wt[(x % D) * D + x / D] = w[x];
  for (int x = t; x < 16 * D; x += 256) {
    const size_t e = ((size_t)bh * D + c0) * D + x;
    float acc = 0.f;
    int sp = 0;
    for (; sp + 4 <= splits; sp += 4) {
      float a[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = m_part[(size_t)(sp + i) * BH * D * D + e];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc += a[i];
    }
    for (; sp < splits; ++sp) acc += m_part[(size_t)sp * BH * D * D + e];
    Ms[x] = acc;
    Ss[x] = S[e];
  }
  if (blk == 0) {
    if (t < D) {
      constexpr int RG = 256 / D;  // row groups of the rows kernel's dz partials
      float acc = 0.f;
      for (int sp = 0; sp < splits; ++sp)
        for (int g = 0; g < RG; ++g) acc += dz_part[(((size_t)sp * BH + bh) * RG + g) * D + t];
      dz[(size_t)bh * D + t] = acc;
    } else if (t == D) {
      float acc = 0.f;
      for (int sp = 0; sp < splits; ++sp) acc += dg_part[(size_t)sp * BH + bh];
      dgate[bh] = acc;
    }
  }
  __syncthreads();
  constexpr int G = 256 / D;     // thread groups: 2 (d = 128) or 4 (d = 64)
  const int col = t % D, grp = t / D;
  // dS rows: thread (e = col, grp) owns rows grp * (16 / G) ...
  {
    constexpr int R = 16 / G;
    float acc[R];
#pragma unroll
    for (int i = 0; i < R; ++i) acc[i] = 0.f;
#pragma unroll 4
    for (int f = 0; f < D; ++f) {
      const float wv = __uint_as_float((uint32_t)Wt[f * D + col] << 16);
#pragma unroll
      for (int i = 0; i < R; ++i) acc[i] = fmaf(Ms[(grp * R + i) * D + f], wv, acc[i]);
    }
#pragma unroll
    for (int i = 0; i < R; ++i) {
      const uint16_t hi = (uint16_t)(pack_bf16x2(acc[i], 0.f) & 0xFFFFu);
      const float rest = acc[i] - __uint_as_float((uint32_t)hi << 16);
      const uint16_t lo = (uint16_t)(pack_bf16x2(rest, 0.f) & 0xFFFFu);
      uint16_t* row = ds_op + ((size_t)bh * D + c0 + grp * R + i) * (2 * D);
      row[col] = hi;
      row[D + col] = lo;
    }
  }
  // S^T M over the 16 rows: thread (f = col, grp) owns e in [grp * D / G, +D / G)
  {
    constexpr int E = D / G;
    float acc[E];
#pragma unroll
    for (int i = 0; i < E; ++i) acc[i] = 0.f;
#pragma unroll 2
    for (int rr = 0; rr < 16; ++rr) {
      const float mv = Ms[rr * D + col];
#pragma unroll
      for (int i = 0; i < E; ++i) acc[i] = fmaf(Ss[rr * D + grp * E + i], mv, acc[i]);
    }
    float* dst = dw_part + (((size_t)bh * (D / 16) + blk) * D + grp * E) * D + col;
#pragma unroll
    for (int i = 0; i < E; ++i) dst[(size_t)i * D] = acc[i];
  }
}

// dW[x] = the partials of lin_state_grad_kernel in (b, h), then row-block order.
__global__ void __launch_bounds__(256) lin_dw_kernel(const float* __restrict__ dw_part, int parts, int DD,
                                                     float* __restrict__ dw) {
  const int x = blockIdx.x * 256 + threadIdx.x;
  if (x >= DD) return;
  float acc = 0.f;
  int p = 0;
  for (; p + 8 <= parts; p += 8) {
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = dw_part[(size_t)(p + i) * DD + x];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc += a[i];
  }
  for (; p < parts; ++p) acc += dw_part[(size_t)p * DD + x];
  dw[x] = acc;
}

template <int D>
cudaError_t launch_rows_t(const LinBwdArgs& a, cudaStream_t s) {
  constexpr int smem = rows_smem<D>();
  cudaError_t e = cudaFuncSetAttribute(lin_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  lin_rows_kernel<D><<<dim3(a.splits, a.B * a.heads), 192, smem, s>>>(
      *a.tm_q, *a.tm_do, *a.tm_t, a.out, a.lse, a.gate, a.z, a.N, a.heads, a.npad, a.tiles_per_split, a.eps, a.dq,
      a.lse2, a.dvec, a.m_part, a.dz_part, a.dg_part, a.status, a.wait_limit_ns);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_tail_t(const LinBwdArgs& a, cudaStream_t s) {
  const int BH = a.B * a.heads;
  const size_t sg_smem = (size_t)32 * D * sizeof(float) + (size_t)D * D * sizeof(uint16_t);
  cudaError_t e = cudaFuncSetAttribute(lin_state_grad_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)sg_smem);
  if (e != cudaSuccess) return e;
  lin_state_grad_kernel<D><<<dim3(BH, D / 16), 256, sg_smem, s>>>(a.m_part, a.dz_part, a.dg_part, a.S, a.w,
                                                                 a.splits, a.ds_op, a.dz, a.dgate, a.dw_part);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lin_dw_kernel<<<(D * D + 255) / 256, 256, 0, s>>>(a.dw_part, BH * (D / 16), D * D, a.dw);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_keys_t(const LinBwdArgs& a, cudaStream_t s) {
  constexpr int smem = keys_smem<D>();
  cudaError_t e = cudaFuncSetAttribute(lin_keys_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  lin_keys_kernel<D><<<dim3(a.splits, a.B * a.heads), 320, smem, s>>>(*a.tm_k, *a.tm_v, *a.tm_ds, a.dz, a.N,
                                                                      a.heads, a.tiles_per_split, a.dk, a.dv,
                                                                      a.status, a.wait_limit_ns);
  return cudaGetLastError();
}

}  // namespace

void linear_backward_splits(int BH, int N, int d, int* splits, int* tiles_per_split) {
  const int ntiles = (N + 127) / 128;
  const int slots = 148 * (d == 128 ? LinBwdCfg<128>::CTAS_PER_SM : LinBwdCfg<64>::CTAS_PER_SM);
  // the fewest splits whose cost (waves x tiles per CTA) is within 5% of the best
  long long best = -1;
  int best_s = 1;
  const int top = ntiles < 512 ? ntiles : 512;
  long long cost[513];
  for (int s = 1; s <= top; ++s) {
    const long long waves = ((long long)BH * s + slots - 1) / slots;
    cost[s] = waves * ((ntiles + s - 1) / s);
    if (best < 0 || cost[s] < best) best = cost[s];
  }
  for (int s = 1; s <= top; ++s)
    if (cost[s] * 100 <= best * 105) {
      best_s = s;
      break;
    }
  const int tps = (ntiles + best_s - 1) / best_s;
  *tiles_per_split = tps;
  *splits = (ntiles + tps - 1) / tps;  // every split owns at least one tile
}

cudaError_t launch_linear_backward_rows(const LinBwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_rows_t<64>(a, s) : launch_rows_t<128>(a, s);
}

cudaError_t launch_linear_backward_state(const LinBwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_tail_t<64>(a, s) : launch_tail_t<128>(a, s);
}

cudaError_t launch_linear_backward_keys(const LinBwdArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_keys_t<64>(a, s) : launch_keys_t<128>(a, s);
}

}  // namespace salad
