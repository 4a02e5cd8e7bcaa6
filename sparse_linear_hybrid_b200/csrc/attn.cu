// SALAD hybrid attention forward: block-sparse softmax attention over the kept
// key blocks (ST-SWA, sciencestack SALAD page Figure 1; the sparse branch of
// SALAD summary section 2.1) fused with the epilogue of the ReLU linear branch,
// its static projection and the per-(b, h) gate (summary sections 2.1-2.3):
//
//   o_sp  = softmax(scale * q K_kept^T) V_kept          (online softmax)
//   o_lin = relu(q)^T S / (relu(q) . z + eps)           (S, z from linear.cu)
//   out   = o_sp + g * (o_lin W);   out = o_sp when g == 0 (branch dropped)
//
// The projection is applied to the state ahead of time (linear.cu hands over
// T = S W), so the linear branch costs one product per query tile:
//   g * (o_lin W) = g * (relu(q) T) / (relu(q) . z + eps).
//
// One CTA owns a 128-row query tile of one (b, h) (two 64-token query blocks
// when block == 64, whose kept-key lists are merged; a key tile then carries a
// bit per half saying which rows may see it).  Warp roles, 352 threads:
//   warp 0     TMA producer: Q once, then K tiles of the kept blocks into a
//              2-deep ring, then (when g != 0) T;
//   warp 10    TMA producer of the V tiles (2-deep ring).  A V stage frees up
//              only when its PV is done; with K and V in one issue order the
//              next K (and so the next S) would wait for that PV as well;
//   warp 1     tcgen05 issuer (one thread) and TMEM owner:
//              S_j = Q K_j^T (A, B in shared memory) into one of two TMEM
//              buffers; O += P_j V_j with P_j read from TMEM; at the end
//              U = relu(Q) T into the S buffer the last tile left free, issued
//              as soon as its operands are in, before or after the last PV;
//   warps 2-9  softmax, two threads per query row (each takes half of the key
//              columns of a tile and half of the feature columns of O): online
//              softmax whose running maximum is only moved (and O rescaled in
//              TMEM) when it grows by more than 2^8, P_j written to TMEM as
//              bf16; after the last tile each thread applies ReLU to its half
//              of its row of Q (the A operand of U) and sums its half of
//              relu(q) . z; finally out = O / l + g U / den and one TMA store
//              of bf16 out.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O [256,256+d),
// P0 [384,448), P1 [448,512) (bf16 pairs).  P is double-buffered: the
// softmax writes P_{j+1} while PV_j still reads P_j, and waits on PV_j only
// when it must rescale O.  Every barrier a role waits on two tiles apart is
// split per buffer, so no wait can fall a phase behind.  T is fed as a hi + lo
// pair of bf16 halves (K doubled, relu(Q) read twice), so U keeps ~16 mantissa
// bits of T.
#include "internal.h"
#include "ptx.cuh"

namespace salad {
namespace {

constexpr uint64_t kDrainNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

struct AttnShared {
  uint64_t q_full;
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2];
  uint64_t t_full, q_relu, u_done;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  uint64_t xbar[4];       // per lane quarter: the two halves of its rows meet here (64 arrivals)
  float xmax[2][2][128];  // per tile parity, per half: partial row maxima
  float xsum[2][128];     // per half: partial row sums
  float xden[2][128];     // per half: partial relu(q) . z
};

template <int D, int BLK>
struct AttnCfg {
  static constexpr int QROWS = 128;
  static constexpr int DCH = D / 64;                // 64-column chunks of a d-wide row
  static constexpr int Q_BYTES = QROWS * D * 2;     // DCH chunks of 16 KB
  static constexpr int KV_BOX = BLK * 128;          // one [BLK x 64] box
  static constexpr int KV_BYTES = DCH * KV_BOX;     // one K or V tile
  static constexpr int RING_BYTES = 4 * KV_BYTES;   // K[2], V[2]
  static constexpr int T_CH = 2 * D / 64;          // 64-column chunks of the [T_hi | T_lo] operand
  static constexpr int T_CH_BYTES = D * 128;        // D rows (feature f) of 128 bytes
  static constexpr int T_BYTES = T_CH * T_CH_BYTES;
  // T goes into the K ring once the last S product has read it when it fits
  // there (d <= block); otherwise it has a region of its own, loaded up front.
  static constexpr bool T_IN_RING = D <= BLK;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = OFF_Q + Q_BYTES;
  static constexpr int OFF_K0 = OFF_RING;
  static constexpr int OFF_V0 = OFF_RING + 2 * KV_BYTES;
  static constexpr int OFF_T = T_IN_RING ? OFF_K0 : OFF_RING + RING_BYTES;
  static constexpr int OFF_BAR = OFF_RING + RING_BYTES + (T_IN_RING ? 0 : T_BYTES);
  static constexpr int SMEM_USED = OFF_BAR + (int)sizeof(AttnShared) + 1024;
  // at least 120 KB so that one CTA (and its 512 TMEM columns) owns the SM
  static constexpr int SMEM = SMEM_USED > 122880 ? SMEM_USED : 122880;
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_P = 384;
  static constexpr uint32_t P_COLS = BLK / 2;       // one P buffer: BLK bf16 per row
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BLK, false, false);   // Q K^T
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);     // P V   (V MN-major)
  static constexpr uint32_t IDESC_U = idesc_bf16(128, D, false, false);     // relu(Q) [T_hi ; T_lo]
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(!T_IN_RING || T_BYTES <= 2 * KV_BYTES, "T must fit the K ring");
  static_assert(TM_P + 2 * P_COLS <= 512 && D <= 128, "tensor memory budget");
};



// Kept key tiles of one 128-row query tile, in ascending key-block order.
// bits: bit s set when query half s (block == 64) or the whole tile uses it.
struct KeyIter {
  const int32_t* a;
  const int32_t* b;
  int na, nb, ia, ib;
  __device__ __forceinline__ bool next(int& col, int& bits) {
    if (ia < na && (ib >= nb || a[ia] <= b[ib])) {
      col = a[ia++];
      bits = 1;
      if (ib < nb && b[ib] == col) {
        bits |= 2;
        ++ib;
      }
      return true;
    }
    if (ib < nb) {
      col = b[ib++];
      bits = 2;
      return true;
    }
    return false;
  }
};

template <int BLK>
__device__ __forceinline__ KeyIter make_iter(const int32_t* row_ptr, const int32_t* col_idx, int h, int nb,
                                             int qtile) {
  KeyIter it{};
  if (BLK == 128) {
    const int r = h * nb + qtile;
    it.a = col_idx + row_ptr[r];
    it.na = row_ptr[r + 1] - row_ptr[r];
    it.b = nullptr;
    it.nb = 0;
  } else {
    const int I0 = 2 * qtile, I1 = 2 * qtile + 1;
    const int r0 = h * nb + I0;
    it.a = col_idx + row_ptr[r0];
    it.na = row_ptr[r0 + 1] - row_ptr[r0];
    if (I1 < nb) {
      it.b = col_idx + row_ptr[r0 + 1];
      it.nb = row_ptr[r0 + 2] - row_ptr[r0 + 1];
    } else {
      it.b = nullptr;
      it.nb = 0;
    }
  }
  it.ia = it.ib = 0;
  return it;
}

__device__ __forceinline__ void record_timeout(AttnShared* sh, uint32_t* status) {
  sh->abort_flag = 1;
  atomicOr(status, kStatusTimeout);
}

__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t x) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0u));
  return r;
}

template <int D, int BLK>
__global__ void __launch_bounds__(352, 1)
    salad_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                      const __grid_constant__ CUtensorMap tm_t, const int32_t* __restrict__ row_ptr,
                      const int32_t* __restrict__ col_idx, const float* __restrict__ gate,
                      const float* __restrict__ zvec, int heads, int N, int qtiles, float scale_log2, float eps,
                      uint32_t* status, uint64_t limit_ns) {
  using C = AttnCfg<D, BLK>;
  const int bh = blockIdx.x / qtiles, qtile = blockIdx.x % qtiles;
  const int b = bh / heads, h = bh % heads;
  const int nb = (N + BLK - 1) / BLK;
  const float g = gate[bh];
  const bool lin = g != 0.0f;  // the linear branch is dropped for this (b, h) when its gate is 0

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnShared* sh = reinterpret_cast<AttnShared*>(smem + C::OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sh->q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh->k_full[s], 1);
      mbar_init(&sh->k_empty[s], 1);
      mbar_init(&sh->v_full[s], 1);
      mbar_init(&sh->v_empty[s], 1);
      mbar_init(&sh->s_full[s], 1);
      mbar_init(&sh->s_free[s], 8);
      mbar_init(&sh->pv_done[s], 1);
      mbar_init(&sh->p_full[s], 8);
    }
    mbar_init(&sh->t_full, 1);
    mbar_init(&sh->q_relu, 8);
    mbar_init(&sh->u_done, 1);
    mbar_init(&sh->drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&sh->xbar[q], 64);
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

  if (warp == 0) {
    // ============================ TMA producer
    int n = 0;
    bool ok = true, t_issued = false;
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_out);
      mbar_arrive_expect_tx(&sh->q_full, C::Q_BYTES);
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch)
        tma_load_3d(smem + C::OFF_Q + ch * 16384, &tm_q, &sh->q_full, h * D + ch * 64, qtile * 128, b);
      auto load_t = [&]() {
        mbar_arrive_expect_tx(&sh->t_full, C::T_BYTES);
#pragma unroll
        for (int ch = 0; ch < C::T_CH; ++ch)
          tma_load_3d(smem + C::OFF_T + ch * C::T_CH_BYTES, &tm_t, &sh->t_full, ch * 64, 0, bh);
        t_issued = true;
      };
      if (lin && !C::T_IN_RING) load_t();
      KeyIter it = make_iter<BLK>(row_ptr, col_idx, h, nb, qtile);
      int col, bits, j = 0;
      while (it.next(col, bits)) {
        const int s = j & 1;
        const uint32_t ph = ((j >> 1) & 1) ^ 1;
        if (sh->abort_flag || !mbar_wait(&sh->k_empty[s], ph, limit_ns)) { ok = false; break; }
        mbar_arrive_expect_tx(&sh->k_full[s], C::KV_BYTES);
        uint8_t* kt = smem + C::OFF_K0 + s * C::KV_BYTES;
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          tma_load_3d(kt + ch * C::KV_BOX, &tm_k, &sh->k_full[s], h * D + ch * 64, col * BLK, b);
        ++j;
      }
      n = j;
      if (ok && lin && C::T_IN_RING) {
        // T overwrites the K ring: wait until the S products have read both stages
        for (int s = 0; s < 2 && ok; ++s) {
          const int uses = (n - s + 1) / 2;
          if (uses > 0) ok = mbar_wait(&sh->k_empty[s], (uint32_t)((uses - 1) & 1), limit_ns);
        }
        if (ok) load_t();
      }
    }
    if (lane == 0) {
      if (!ok) record_timeout(sh, status);
      // every copy this thread started lands before the CTA may exit (at once
      // unless another role gave up early)
      mbar_wait(&sh->q_full, 0, kDrainNs);
      for (int i = (n > 2 ? n - 2 : 0); i < n; ++i) mbar_wait(&sh->k_full[i & 1], (i >> 1) & 1, kDrainNs);
      if (t_issued) mbar_wait(&sh->t_full, 0, kDrainNs);
    }
  } else if (warp == 10) {
    // ============================ TMA producer of the V tiles
    if (lane == 0) {
      tma_prefetch_map(&tm_v);
      KeyIter it = make_iter<BLK>(row_ptr, col_idx, h, nb, qtile);
      int col, bits, j = 0;
      bool ok = true;
      while (it.next(col, bits)) {
        const int s = j & 1;
        if (sh->abort_flag || !mbar_wait(&sh->v_empty[s], ((j >> 1) & 1) ^ 1, limit_ns)) { ok = false; break; }
        mbar_arrive_expect_tx(&sh->v_full[s], C::KV_BYTES);
        uint8_t* vt = smem + C::OFF_V0 + s * C::KV_BYTES;
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          tma_load_3d(vt + ch * C::KV_BOX, &tm_v, &sh->v_full[s], h * D + ch * 64, col * BLK, b);
        ++j;
      }
      if (!ok) record_timeout(sh, status);
      for (int i = (j > 2 ? j - 2 : 0); i < j; ++i) mbar_wait(&sh->v_full[i & 1], (i >> 1) & 1, kDrainNs);
    }
  } else if (warp == 1) {
    // ============================ tcgen05 issuer
    if (lane == 0) {
      bool ok = mbar_wait(&sh->q_full, 0, limit_ns);
      const uint32_t q_addr = sbase + C::OFF_Q;
      KeyIter it = make_iter<BLK>(row_ptr, col_idx, h, nb, qtile);
      int col, bits, j = 0;
      // O += P_i V_i, P_i from tensor memory (operands already waited for)
      auto issue_pv_now = [&](int i) {
        const int s = i & 1;
        tc_fence_after();
        const uint32_t vt = sbase + C::OFF_V0 + s * C::KV_BYTES;
        const uint32_t pt = tmem + C::TM_P + s * C::P_COLS;
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk) {
          const uint64_t bd = sw128_desc(vt + kk * 2048, C::KV_BOX, 1024);
          mma_bf16_ts(tmem + C::TM_O, pt + kk * 8, bd, C::IDESC_PV, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sh->pv_done[s]);
        mma_commit(&sh->v_empty[s]);
      };
      auto issue_pv = [&](int i) -> bool {
        const int s = i & 1;
        if (sh->abort_flag || !mbar_wait(&sh->p_full[s], (uint32_t)((i >> 1) & 1), limit_ns)) return false;
        if (!mbar_wait(&sh->v_full[s], (uint32_t)((i >> 1) & 1), limit_ns)) return false;
        issue_pv_now(i);
        return true;
      };
      while (ok && it.next(col, bits)) {
        const int s = j & 1;
        if (sh->abort_flag || !mbar_wait(&sh->k_full[s], (uint32_t)((j >> 1) & 1), limit_ns)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&sh->s_free[s], (uint32_t)(((j - 2) >> 1) & 1), limit_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t kt = sbase + C::OFF_K0 + s * C::KV_BYTES;
        const uint32_t d_s = tmem + (s ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sw128_desc(q_addr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(kt + (kk / 4) * C::KV_BOX + (kk % 4) * 32, 16, 1024);
          mma_bf16_ss(d_s, a, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sh->s_full[s]);
        mma_commit(&sh->k_empty[s]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; ++j; break; }
        ++j;
      }
      // The last PV and U = relu(Q) [T_hi ; T_lo] (K = 2d: relu(Q) is fed twice)
      // go in whichever order their operands arrive.  U lands in the S buffer
      // of tile n, whose previous user S_{n-2} the softmax has read by then.
      const int n = j;
      bool pv_left = ok && n >= 1, u_left = ok && lin;
      const int sl = (n - 1) & 1, ub = n & 1;
      const uint32_t ph_l = (uint32_t)(((n - 1) >> 1) & 1), ph_u = (uint32_t)(((n - 2) >> 1) & 1);
      const uint64_t t0 = global_timer_ns();
      while (pv_left || u_left) {
        if (pv_left && mbar_try_wait(&sh->p_full[sl], ph_l) && mbar_try_wait(&sh->v_full[sl], ph_l)) {
          issue_pv_now(n - 1);
          pv_left = false;
        } else if (u_left && mbar_try_wait(&sh->t_full, 0) && mbar_try_wait(&sh->q_relu, 0) &&
                   (n < 2 || mbar_try_wait(&sh->s_free[ub], ph_u))) {
          tc_fence_after();
          const uint32_t tb = sbase + C::OFF_T;
#pragma unroll
          for (int kk = 0; kk < 2 * D / 16; ++kk) {
            const int qk = kk % (D / 16);
            const uint64_t a = sw128_desc(q_addr + (qk / 4) * 16384 + (qk % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(tb + (kk / 4) * C::T_CH_BYTES + (kk % 4) * 32, 16, 1024);
            mma_bf16_ss(tmem + (ub ? C::TM_S1 : C::TM_S0), a, bd, C::IDESC_U, kk > 0 ? 1u : 0u);
          }
          mma_commit(&sh->u_done);
          u_left = false;
        } else if (sh->abort_flag || global_timer_ns() - t0 > limit_ns) {
          ok = false;
          break;
        }
      }
      if (!ok) {
        record_timeout(sh, status);
        mma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kDrainNs);
      }
    }
  } else {
    // ============================ softmax / epilogue (warps 2..9): two threads per query row
    // Warps w and w+4 sit on the same TMEM lane quarter (w & 3) and own the same
    // 32 query rows; hf = 0 takes key columns [0, BLK/2) and feature columns
    // [0, D/2), hf = 1 the other halves.  The two halves exchange their partial
    // row maxima through shared memory each tile, so both take the same
    // (running-max, rescale) decision; partial row sums are combined once at the end.
    constexpr int HC = BLK / 2;                               // key columns per thread
    constexpr int HD = D / 2;                                 // feature columns per thread
    const int sw = warp - 2;
    const int hf = sw >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                        // query row within the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int half = BLK == 64 ? (r >> 6) : 0;               // query half (block 64), warp-uniform
    const uint32_t q_addr = sbase + C::OFF_Q;
    const uint64_t c2 = f32x2_pack(scale_log2, scale_log2);
    float m_ref = -INFINITY;  // running reference max (raw score units), same in both halves
    float l = 0.f;            // this half's share of the row sum
    bool ok = true;
    float gd = 0.f;           // g / (relu(q) . z + eps), the linear branch's row factor
    KeyIter it = make_iter<BLK>(row_ptr, col_idx, h, nb, qtile);
    int col, bits, j = 0;
    while (ok && it.next(col, bits)) {
      const int s = j & 1;
      const bool aborted = __shfl_sync(0xffffffffu, sh->abort_flag != 0, 0);
      if (aborted || !mbar_wait_warp(&sh->s_full[s], (uint32_t)((j >> 1) & 1), limit_ns)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[HC];
#pragma unroll
      for (int c = 0; c < HC / 32; ++c)
        tmem_ld32(lane_addr + (s ? C::TM_S1 : C::TM_S0) + hf * HC + c * 32,
                  *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]));
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->s_free[s]);

      const bool use = ((bits >> half) & 1) != 0;      // warp-uniform
      const int valid = min(BLK, N - col * BLK) - hf * HC;  // real keys among this thread's columns
      float mt;
      if (valid >= HC) {
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int i = 0; i < HC; i += 8) {
          m0 = fmax3(m0, __uint_as_float(sr[i + 0]), __uint_as_float(sr[i + 1]));
          m1 = fmax3(m1, __uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3]));
          m2 = fmax3(m2, __uint_as_float(sr[i + 4]), __uint_as_float(sr[i + 5]));
          m3 = fmax3(m3, __uint_as_float(sr[i + 6]), __uint_as_float(sr[i + 7]));
        }
        mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
      } else {
        // partial last block: keys past N never count (valid may be <= 0 here)
#pragma unroll
        for (int i = 0; i < HC; ++i)
          if (i >= valid) sr[i] = __float_as_uint(-INFINITY);
        float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
        for (int i = 0; i < HC; i += 4) {
          m0 = fmax3(m0, __uint_as_float(sr[i + 0]), __uint_as_float(sr[i + 1]));
          m1 = fmax3(m1, __uint_as_float(sr[i + 2]), __uint_as_float(sr[i + 3]));
        }
        mt = fmaxf(m0, m1);
      }
      // both halves of the row agree on the tile maximum (one barrier phase per tile;
      // a bounded wait, so a time-out on either side cannot hang its partner)
      sh->xmax[j & 1][hf][r] = mt;
      mbar_arrive(&sh->xbar[quarter]);
      if (!mbar_wait_warp(&sh->xbar[quarter], (uint32_t)(j & 1), limit_ns)) { ok = false; break; }
      mt = fmaxf(mt, sh->xmax[j & 1][hf ^ 1][r]);
      float alpha = 1.f;
      bool rescale = false;
      if (use) {
        if (m_ref == -INFINITY) {
          m_ref = mt;
        } else if ((mt - m_ref) * scale_log2 > kRescaleThreshold) {
          alpha = ex2_approx((m_ref - mt) * scale_log2);
          m_ref = mt;
          rescale = true;
        }
      }
      // p = 2^(s * c - m_ref * c) in pairs; rows that do not use the tile write zeros
      uint32_t pk[HC / 2];
      float rs;
      {
        const uint64_t nmb2 = f32x2_pack(-m_ref * scale_log2, -m_ref * scale_log2);
        uint64_t acc0 = 0, acc1 = 0, acc2 = 0, acc3 = 0;  // 0.0f pairs
#pragma unroll
        for (int i = 0; i < HC / 2; ++i) {
          const uint64_t x = f32x2_fma(f32x2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, nmb2);
          float p0, p1;
          if ((i & 3) == 3) {
            // one pair in four on the FMA pipe, relieving the special-function unit
            exp2_fma_x2(x, p0, p1);
          } else {
            float x0, x1;
            f32x2_unpack(x, x0, x1);
            p0 = ex2_approx(x0);
            p1 = ex2_approx(x1);
          }
          const uint64_t pp = f32x2_pack(p0, p1);
          if ((i & 3) == 0) acc0 = f32x2_add(acc0, pp);
          if ((i & 3) == 1) acc1 = f32x2_add(acc1, pp);
          if ((i & 3) == 2) acc2 = f32x2_add(acc2, pp);
          if ((i & 3) == 3) acc3 = f32x2_add(acc3, pp);
          pk[i] = pack_bf16x2(p0, p1);
        }
        const uint64_t a = f32x2_add(f32x2_add(acc0, acc1), f32x2_add(acc2, acc3));
        float a0, a1;
        f32x2_unpack(a, a0, a1);
        rs = a0 + a1;
      }
      if (!use) {
#pragma unroll
        for (int i = 0; i < HC / 2; ++i) pk[i] = 0u;
        rs = 0.f;
      }
      l = l * alpha + rs;
      // P buffer s was last read by PV_{j-2}; O may be rescaled only after PV_{j-1}
      if (j >= 2) {
        if (!mbar_wait_warp(&sh->pv_done[s], (uint32_t)(((j - 2) >> 1) & 1), limit_ns)) { ok = false; break; }
      }
      if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
        if (!mbar_wait_warp(&sh->pv_done[s ^ 1], (uint32_t)(((j - 1) >> 1) & 1), limit_ns)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(lane_addr + C::TM_O + hf * HD + c * 32, rr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32(lane_addr + C::TM_O + hf * HD + c * 32, rr);
        }
      }
      tc_fence_after();
      if constexpr (HC / 2 == 32) {
        tmem_st32(lane_addr + C::TM_P + s * C::P_COLS + hf * (HC / 2), *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
      } else {
        tmem_st16(lane_addr + C::TM_P + s * C::P_COLS + hf * (HC / 2), *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->p_full[s]);
      ++j;
    }
    const int n = j;
    float den_h = 0.f;  // relu(q) . z over this half of the row
    if (ok && lin) ok = mbar_wait_warp(&sh->q_full, 0, limit_ns);  // (no S product read Q when n == 0)
    if (ok && lin) {
      // relu(Q) in place for U, each thread its half of its row (the S products
      // are done with Q: the last one completed before this thread read its S),
      // and this half's share of relu(q) . z on the way
      const float4* zr = reinterpret_cast<const float4*>(zvec + (size_t)bh * D);
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int t = 0; t < C::DCH * 4; ++t) {
        const int piece = hf * C::DCH * 4 + t;  // 16-byte piece of the row: features 8 * piece ...
        const uint32_t addr = q_addr + (piece / 8) * 16384 + sw128_offset((uint32_t)r, (uint32_t)(piece % 8));
        uint32_t x[4];
        ld_shared_v4(addr, x[0], x[1], x[2], x[3]);
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = relu_bf16x2(x[i]);
        st_shared_v4(addr, x[0], x[1], x[2], x[3]);
        const float4 za = __ldg(zr + piece * 2), zb = __ldg(zr + piece * 2 + 1);
        const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          d0 = fmaf(bf16_lo_to_f32(x[i]), zz[2 * i], d0);
          d1 = fmaf(bf16_hi_to_f32(x[i]), zz[2 * i + 1], d1);
        }
      }
      den_h = d0 + d1;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->q_relu);
    }
    if (ok && n >= 1) {
      ok = mbar_wait_warp(&sh->pv_done[(n - 1) & 1], (uint32_t)(((n - 1) >> 1) & 1), limit_ns);
      tc_fence_after();
    }
    // the row sum of both halves (barrier phase n)
    if (ok) {
      sh->xsum[hf][r] = l;
      sh->xden[hf][r] = den_h;
      mbar_arrive(&sh->xbar[quarter]);
      ok = mbar_wait_warp(&sh->xbar[quarter], (uint32_t)(n & 1), limit_ns);
      if (ok) {
        l += sh->xsum[hf ^ 1][r];
        if (lin) gd = g / ((sh->xden[0][r] + sh->xden[1][r]) + eps);  // same order in both halves
      }
    }
    if (ok) ok = mbar_wait_warp(&sh->q_full, 0, limit_ns);  // the staging area below is the Q tile
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    // U has read relu(Q) once u_done completes, so the Q tile is free for staging
    if (ok && lin) ok = mbar_wait_warp(&sh->u_done, 0, limit_ns);
    if (ok) {
      tc_fence_after();
      // out = O / l + g U / den for this half's features -> bf16 staging in the Q tile
      const uint32_t tm_u = (n & 1) ? C::TM_S1 : C::TM_S0;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t ro[32], ru[32];
        if (n >= 1) {
          tmem_ld32(lane_addr + C::TM_O + hf * HD + c * 32, ro);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ro[i] = 0u;
        }
        if (lin) {
          tmem_ld32(lane_addr + tm_u + hf * HD + c * 32, ru);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ru[i] = 0u;
        }
        tmem_ld_wait();
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float o0 = fmaf(gd, __uint_as_float(ru[2 * i]), __uint_as_float(ro[2 * i]) * inv_l);
          const float o1 = fmaf(gd, __uint_as_float(ru[2 * i + 1]), __uint_as_float(ro[2 * i + 1]) * inv_l);
          packed[i] = pack_bf16x2(o0, o1);
        }
        const int f0 = hf * HD + c * 32;  // first feature of these 32 columns
        const int ch = f0 / 64, pc0 = (f0 % 64) / 8;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          st_shared_v4(q_addr + ch * 16384 + sw128_offset((uint32_t)r, (uint32_t)(pc0 + k)), packed[4 * k],
                       packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
      }
      fence_proxy_async_smem();
    } else {
      record_timeout(sh, status);
    }
    named_bar_sync(1, 256);
    if (threadIdx.x == 64 && !sh->abort_flag) {
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch)
        tma_store_3d(&tm_out, smem + C::OFF_Q + ch * 16384, h * D + ch * 64, qtile * 128, b);
      bulk_commit_group();
      bulk_wait_group_read0();
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

template <int D, int BLK>
cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t s) {
  using C = AttnCfg<D, BLK>;
  cudaError_t e =
      cudaFuncSetAttribute(salad_attn_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int qtiles = (a.N + 127) / 128;
  const long long grid = (long long)qtiles * a.B * a.heads;
  salad_attn_kernel<D, BLK><<<(unsigned)grid, 352, C::SMEM, s>>>(
      *a.tm_q, *a.tm_k, *a.tm_v, *a.tm_out, *a.tm_t, a.row_ptr, a.col_idx, a.gate, a.z, a.heads, a.N, qtiles,
      a.scale_log2, a.eps, a.status, a.wait_limit_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  if (a.d == 64) return a.block == 64 ? launch_attn_t<64, 64>(a, s) : launch_attn_t<64, 128>(a, s);
  return a.block == 64 ? launch_attn_t<128, 64>(a, s) : launch_attn_t<128, 128>(a, s);
}

}  // namespace salad
