// SALAD hybrid attention forward: block-sparse softmax attention over the kept
// key blocks (ST-SWA, sciencestack SALAD page Figure 1; the sparse branch of
// SALAD summary section 2.1) fused with the epilogue of the ReLU linear branch,
// its static projection and the per-(b, h) gate (summary sections 2.1-2.3):
//
//   o_sp  = softmax(scale * q K_kept^T) V_kept          (online softmax)
//   o_lin = relu(q)^T S / (relu(q) . z + eps)           (S, z from linear.cu)
//   out   = o_sp + g * (o_lin W);   out = o_sp when g == 0 (branch dropped)
//
// One CTA owns a 128-row query tile of one (b, h) (two 64-token query blocks
// when block == 64, whose kept-key lists are merged; a key tile then carries a
// bit per half saying which rows may see it).  Two CTAs share an SM (about
// 97 KB of shared memory and 256 tensor-memory columns each), so one CTA's
// softmax, MMAs, loads and epilogue overlap the other's.  160 threads:
//   warp 0, lane 0   control: TMA loads (Q once, then the K and V tile of each
//                    kept block, single-buffered) and the tcgen05 MMAs
//                    S_j = Q K_j^T and O += P_j V_j;  warp 0 owns the TMEM;
//   warps 1-4        softmax, one query row per thread: online softmax whose
//                    running maximum only moves (and O is only rescaled) when
//                    it grows by more than 2^8; P_j is written as bf16 into the
//                    first columns of S_j's own tensor memory; then the fused
//                    epilogue and one TMA store of bf16 out.
// Tensor memory: S [0, block) (P aliased on its first block/2 columns),
// O [128, 128+d).  Epilogue (g != 0): U = relu(Q) [S_hi ; S_lo] lands on [0, d),
// the softmax warps replace it by o' = (l g / (relu(q).z + eps)) U as bf16
// hi + lo halves, and O += [o'_hi | o'_lo] [W ; W] accumulates the projected
// linear branch into O, so out = O / l.  [S|z] and o' are split into hi + lo
// bf16 pairs (K doubled), keeping ~16 mantissa bits in the epilogue products.
#include "internal.h"
#include "ptx.cuh"

namespace salad {
namespace {

constexpr uint64_t kDrainNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8

template <int D, int BLK>
struct AttnCfg {
  static constexpr int DCH = D / 64;               // 64-column chunks of a d-wide row
  static constexpr int Q_BYTES = 128 * D * 2;      // DCH chunks of 16 KB
  static constexpr int KV_BOX = BLK * 128;         // one [BLK x 64] box
  static constexpr int KV_BYTES = DCH * KV_BOX;    // one K or V tile
  static constexpr int SZ_CH = 2 * D / 64;         // K chunks of [S_hi ; S_lo]^T (d rows each)
  static constexpr int SZ_CH_BYTES = D * 128;
  static constexpr int SZ_BYTES = SZ_CH * SZ_CH_BYTES;
  static constexpr int W_CH_BYTES = D * 128;
  static constexpr int W_BYTES = DCH * W_CH_BYTES;
  static constexpr int OVL_BYTES = 2 * KV_BYTES > SZ_BYTES ? 2 * KV_BYTES : SZ_BYTES;
  static constexpr int OFF_Q = 0;                  // Q; relu(Q) in the epilogue; then W
  static constexpr int OFF_K = Q_BYTES;            // K and V tiles; [S|z] operand; out staging
  static constexpr int OFF_V = OFF_K + KV_BYTES;
  static constexpr int OFF_SZ = OFF_K;
  static constexpr int OFF_W = OFF_Q;
  static constexpr int OFF_BAR = OFF_K + OVL_BYTES;
  static constexpr int SMEM = OFF_BAR + 256 + 1024;
  static constexpr uint32_t TM_S = 0, TM_O = 128, TM_U = 0, TM_OL = 0;
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BLK, false, false);  // Q K^T
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);    // P V   (V MN-major)
  static constexpr uint32_t IDESC_U = idesc_bf16(128, D, false, false);    // relu(Q) [S_hi ; S_lo]
  static constexpr uint32_t IDESC_Y = idesc_bf16(128, D, false, true);     // o' W   (W MN-major)
  static_assert(W_BYTES <= Q_BYTES, "W reuses the Q tile");
  static_assert(SMEM <= 113 * 1024, "two CTAs per SM");
};

struct AttnShared {
  uint64_t q_full, k_full, v_full, k_free;
  uint64_t s_full, p_full, pv_done;
  uint64_t sz_full, q_relu, u_done, w_full, a2_full, y_done;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
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

__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t x) { return x & ~(((x >> 15) & 0x00010001u) * 0xFFFFu); }

template <int D, int BLK>
__global__ void __launch_bounds__(160, 2)
    salad_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                      const __grid_constant__ CUtensorMap tm_sz, const __grid_constant__ CUtensorMap tm_w,
                      const int32_t* __restrict__ row_ptr, const int32_t* __restrict__ col_idx,
                      const float* __restrict__ gate, const uint16_t* __restrict__ sz, int heads, int N,
                      int qtiles, float scale_log2, float eps, uint32_t* status, uint64_t limit_ns) {
  using C = AttnCfg<D, BLK>;
  const int bh = blockIdx.x / qtiles, qtile = blockIdx.x % qtiles;
  const int b = bh / heads, h = bh % heads;
  const int nb = (N + BLK - 1) / BLK;
  const float g = gate[bh];

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnShared* sh = reinterpret_cast<AttnShared*>(smem + C::OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&sh->q_full, 1);
    mbar_init(&sh->k_full, 1);
    mbar_init(&sh->v_full, 1);
    mbar_init(&sh->k_free, 1);
    mbar_init(&sh->s_full, 1);
    mbar_init(&sh->p_full, 4);
    mbar_init(&sh->pv_done, 1);
    mbar_init(&sh->sz_full, 1);
    mbar_init(&sh->q_relu, 4);
    mbar_init(&sh->u_done, 1);
    mbar_init(&sh->w_full, 1);
    mbar_init(&sh->a2_full, 4);
    mbar_init(&sh->y_done, 1);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sh->tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ============================ control: TMA + tcgen05 (one thread)
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      tma_prefetch_map(&tm_v);
      tma_prefetch_map(&tm_out);
      const uint32_t q_addr = sbase + C::OFF_Q, k_addr = sbase + C::OFF_K, v_addr = sbase + C::OFF_V;
      KeyIter it = make_iter<BLK>(row_ptr, col_idx, h, nb, qtile);
      int col, bits, ncol, nbits;
      bool have = it.next(col, bits);
      // TMA bookkeeping for the drain on time-out
      int k_issued = 0, v_issued = 0, ep_issued = 0;
      mbar_arrive_expect_tx(&sh->q_full, C::Q_BYTES);
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch)
        tma_load_3d(smem + C::OFF_Q + ch * 16384, &tm_q, &sh->q_full, h * D + ch * 64, qtile * 128, b);
      if (have) {
        mbar_arrive_expect_tx(&sh->k_full, C::KV_BYTES);
        mbar_arrive_expect_tx(&sh->v_full, C::KV_BYTES);
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch) {
          tma_load_3d(smem + C::OFF_K + ch * C::KV_BOX, &tm_k, &sh->k_full, h * D + ch * 64, col * BLK, b);
          tma_load_3d(smem + C::OFF_V + ch * C::KV_BOX, &tm_v, &sh->v_full, h * D + ch * 64, col * BLK, b);
        }
        k_issued = v_issued = 1;
      }
      bool ok = mbar_wait(&sh->q_full, 0, limit_ns);
      int j = 0;
      while (ok && have) {
        const uint32_t ph = (uint32_t)(j & 1);
        const bool more = it.next(ncol, nbits);
        // S_j = Q K_j^T   (the S/P columns are free: PV_{j-1} was awaited below)
        if (sh->abort_flag || !mbar_wait(&sh->k_full, ph, limit_ns)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t a = sw128_desc(q_addr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(k_addr + (kk / 4) * C::KV_BOX + (kk % 4) * 32, 16, 1024);
          mma_bf16_ss(tmem + C::TM_S, a, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sh->s_full);
        mma_commit(&sh->k_free);
        // K_{j+1} may overwrite K_j once S_j is done
        if (!mbar_wait(&sh->k_free, ph, limit_ns)) { ok = false; break; }
        if (more) {
          mbar_arrive_expect_tx(&sh->k_full, C::KV_BYTES);
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_3d(smem + C::OFF_K + ch * C::KV_BOX, &tm_k, &sh->k_full, h * D + ch * 64, ncol * BLK, b);
          ++k_issued;
        }
        // O += P_j V_j  (P_j from tensor memory, on S_j's columns)
        if (sh->abort_flag || !mbar_wait(&sh->p_full, ph, limit_ns) || !mbar_wait(&sh->v_full, ph, limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk) {
          const uint64_t bd = sw128_desc(v_addr + kk * 2048, C::KV_BOX, 1024);
          mma_bf16_ts(tmem + C::TM_O, tmem + C::TM_S + kk * 8, bd, C::IDESC_PV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sh->pv_done);
        // V_{j+1} may overwrite V_j, and S_{j+1} may overwrite P_j, once PV_j is done
        if (!mbar_wait(&sh->pv_done, ph, limit_ns)) { ok = false; break; }
        if (more) {
          mbar_arrive_expect_tx(&sh->v_full, C::KV_BYTES);
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_3d(smem + C::OFF_V + ch * C::KV_BOX, &tm_v, &sh->v_full, h * D + ch * 64, ncol * BLK, b);
          ++v_issued;
        }
        col = ncol;
        bits = nbits;
        have = more;
        ++j;
      }
      if (ok && g != 0.0f) {
        // U = relu(Q) [S_hi ; S_lo]  (K = 2d: relu(Q) is fed twice), into S's columns
        mbar_arrive_expect_tx(&sh->sz_full, C::SZ_BYTES);
#pragma unroll
        for (int ch = 0; ch < C::SZ_CH; ++ch)
          tma_load_3d(smem + C::OFF_SZ + ch * C::SZ_CH_BYTES, &tm_sz, &sh->sz_full, ch * 64, 0, bh);
        ep_issued = 1;
        ok = mbar_wait(&sh->q_relu, 0, limit_ns) && mbar_wait(&sh->sz_full, 0, limit_ns);
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 2 * D / 16; ++kk) {
            const int qk = kk % (D / 16);
            const uint64_t a = sw128_desc(q_addr + (qk / 4) * 16384 + (qk % 4) * 32, 16, 1024);
            const uint64_t bd = sw128_desc(sbase + C::OFF_SZ + (kk / 4) * C::SZ_CH_BYTES + (kk % 4) * 32, 16, 1024);
            mma_bf16_ss(tmem + C::TM_U, a, bd, C::IDESC_U, kk > 0 ? 1u : 0u);
          }
          mma_commit(&sh->u_done);
          // W replaces relu(Q) once U is done
          ok = mbar_wait(&sh->u_done, 0, limit_ns);
        }
        if (ok) {
          mbar_arrive_expect_tx(&sh->w_full, C::W_BYTES);
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_2d(smem + C::OFF_W + ch * C::W_CH_BYTES, &tm_w, &sh->w_full, ch * 64, 0);
          ep_issued = 2;
          // O += [o'_hi | o'_lo] [W ; W]   (o' from tensor memory)
          ok = mbar_wait(&sh->a2_full, 0, limit_ns) && mbar_wait(&sh->w_full, 0, limit_ns);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 2 * D / 16; ++kk) {
              const uint64_t bd = sw128_desc(sbase + C::OFF_W + (kk % (D / 16)) * 2048, C::W_CH_BYTES, 1024);
              mma_bf16_ts(tmem + C::TM_O, tmem + C::TM_OL + kk * 8, bd, C::IDESC_Y, (j > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(&sh->y_done);
          }
        }
      }
      if (!ok) {
        record_timeout(sh, status);
        // let every copy and MMA this thread started finish before the CTA can exit
        mma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kDrainNs);
        mbar_wait(&sh->q_full, 0, kDrainNs);
        if (k_issued > 0) mbar_wait(&sh->k_full, (uint32_t)((k_issued - 1) & 1), kDrainNs);
        if (v_issued > 0) mbar_wait(&sh->v_full, (uint32_t)((v_issued - 1) & 1), kDrainNs);
        if (ep_issued >= 1) mbar_wait(&sh->sz_full, 0, kDrainNs);
        if (ep_issued >= 2) mbar_wait(&sh->w_full, 0, kDrainNs);
      }
    }
  } else {
    // ============================ softmax / epilogue (warps 1..4)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                        // query row within the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int half = BLK == 64 ? (r >> 6) : 0;               // uniform within a warp
    const uint32_t q_addr = sbase + C::OFF_Q;
    const uint64_t c2 = f32x2_pack(scale_log2, scale_log2);
    float m_ref = -INFINITY;  // running reference max (raw score units)
    float l = 0.f;
    bool ok = true;
    KeyIter it = make_iter<BLK>(row_ptr, col_idx, h, nb, qtile);
    int col, bits, j = 0;
    while (it.next(col, bits)) {
      const uint32_t ph = (uint32_t)(j & 1);
      const bool aborted = __shfl_sync(0xffffffffu, sh->abort_flag != 0, 0);
      if (aborted || !mbar_wait_warp(&sh->s_full, ph, limit_ns)) { ok = false; break; }
      tc_fence_after();
      const bool use = ((bits >> half) & 1) != 0;      // warp-uniform
      const int valid = min(BLK, N - col * BLK);       // real keys in this block (warp-uniform)
      const uint32_t s_addr = lane_addr + C::TM_S;
      // pass 1: tile maximum, 64 columns at a time, independent 3-input max chains
      float mt;
      {
        float m0 = -INFINITY, m1 = -INFINITY, m2 = -INFINITY, m3 = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < BLK / 64; ++hh) {
          uint32_t ra[32], rb[32];
          tmem_ld32(s_addr + hh * 64, ra);
          tmem_ld32(s_addr + hh * 64 + 32, rb);
          tmem_ld_wait();
          if (valid < BLK) {  // partial last block: keys past N never count
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              if (hh * 64 + i >= valid) ra[i] = __float_as_uint(-INFINITY);
              if (hh * 64 + 32 + i >= valid) rb[i] = __float_as_uint(-INFINITY);
            }
          }
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            m0 = fmax3(m0, __uint_as_float(ra[i + 0]), __uint_as_float(ra[i + 1]));
            m1 = fmax3(m1, __uint_as_float(ra[i + 2]), __uint_as_float(ra[i + 3]));
            m2 = fmax3(m2, __uint_as_float(rb[i + 0]), __uint_as_float(rb[i + 1]));
            m3 = fmax3(m3, __uint_as_float(rb[i + 2]), __uint_as_float(rb[i + 3]));
          }
        }
        mt = fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
      }
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
      // pass 2: p = 2^(s * c - m_ref * c) in pairs, 64 columns at a time; P goes
      // as bf16 pairs over S_j's first block/2 columns (this lane's row only:
      // columns [32hh, 32hh+32) were read before they are rewritten); rows that
      // do not use the tile write zeros
      float rs;
      {
        const uint64_t nmb2 = f32x2_pack(-m_ref * scale_log2, -m_ref * scale_log2);
        uint64_t acc0 = 0, acc1 = 0, acc2 = 0, acc3 = 0;  // 0.0f pairs
#pragma unroll
        for (int hh = 0; hh < BLK / 64; ++hh) {
          uint32_t ra[32], rb[32];
          tmem_ld32(s_addr + hh * 64, ra);
          tmem_ld32(s_addr + hh * 64 + 32, rb);
          tmem_ld_wait();
          uint32_t pk[32];
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const uint32_t* src = k < 16 ? ra : rb;
            const int e = (k % 16) * 2;
            const uint64_t x = f32x2_fma(f32x2_pack(__uint_as_float(src[e]), __uint_as_float(src[e + 1])), c2, nmb2);
            float x0, x1;
            f32x2_unpack(x, x0, x1);
            float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
            if (valid < BLK) {
              const int cidx = hh * 64 + 2 * k;
              if (cidx >= valid) p0 = 0.f;
              if (cidx + 1 >= valid) p1 = 0.f;
            }
            const uint64_t pp = f32x2_pack(p0, p1);
            if ((k & 3) == 0) acc0 = f32x2_add(acc0, pp);
            if ((k & 3) == 1) acc1 = f32x2_add(acc1, pp);
            if ((k & 3) == 2) acc2 = f32x2_add(acc2, pp);
            if ((k & 3) == 3) acc3 = f32x2_add(acc3, pp);
            pk[k] = use ? pack_bf16x2(p0, p1) : 0u;
          }
          tmem_st32(s_addr + hh * 32, pk);
        }
        const uint64_t acc = f32x2_add(f32x2_add(acc0, acc1), f32x2_add(acc2, acc3));
        float a0, a1;
        f32x2_unpack(acc, a0, a1);
        rs = use ? a0 + a1 : 0.f;
      }
      l = l * alpha + rs;
      // O holds PV_0 .. PV_{j-1} (all complete: S_j was issued after PV_{j-1} finished)
      if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          tmem_ld32(lane_addr + C::TM_O + c * 32, rr);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) rr[i] = __float_as_uint(__uint_as_float(rr[i]) * alpha);
          tmem_st32(lane_addr + C::TM_O + c * 32, rr);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->p_full);
      ++j;
    }
    const int n = j;
    if (ok && n >= 1) {
      ok = mbar_wait_warp(&sh->pv_done, (uint32_t)((n - 1) & 1), limit_ns);
      tc_fence_after();
    }
    if (ok) ok = mbar_wait_warp(&sh->q_full, 0, limit_ns);
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const bool lin = ok && g != 0.0f;
    float den = 0.f;
    if (lin) {
      // relu(Q) in place (the S MMAs are done with Q); den = relu(q) . z with
      // z = z_hi + z_lo from row d of the [S|z] operand in global memory
      const uint16_t* zrow = sz + ((size_t)bh * (D + 16) + D) * (2 * D);
      float d0 = 0.f, d1 = 0.f;
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch)
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t addr = q_addr + ch * 16384 + sw128_offset((uint32_t)r, (uint32_t)c);
          uint32_t x[4];
          ld_shared_v4(addr, x[0], x[1], x[2], x[3]);
#pragma unroll
          for (int k = 0; k < 4; ++k) x[k] = relu_bf16x2(x[k]);
          st_shared_v4(addr, x[0], x[1], x[2], x[3]);
          const int f0 = ch * 64 + c * 8;  // first feature of this 16-byte piece
          const uint4 zh = __ldg(reinterpret_cast<const uint4*>(zrow + f0));
          const uint4 zl = __ldg(reinterpret_cast<const uint4*>(zrow + D + f0));
          const uint32_t zhw[4] = {zh.x, zh.y, zh.z, zh.w}, zlw[4] = {zl.x, zl.y, zl.z, zl.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float z0 = bf16_lo_to_f32(zhw[k]) + bf16_lo_to_f32(zlw[k]);
            const float z1 = bf16_hi_to_f32(zhw[k]) + bf16_hi_to_f32(zlw[k]);
            d0 = fmaf(bf16_lo_to_f32(x[k]), z0, d0);
            d1 = fmaf(bf16_hi_to_f32(x[k]), z1, d1);
          }
        }
      den = d0 + d1;
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->q_relu);
    }
    bool lin_ok = lin && mbar_wait_warp(&sh->u_done, 0, limit_ns);
    if (lin && !lin_ok) ok = false;
    if (lin_ok) {
      tc_fence_after();
      // o' = (l g / (den + eps)) U, as bf16 hi + lo halves over U's own columns
      // (32 columns of U at a time; each piece is read before its columns are
      // rewritten, since o'_hi of columns [32c, 32c+32) lands on [16c, 16c+16))
      const float sc = l * g / (den + eps);
      uint32_t ra[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(lane_addr + C::TM_U + c * 32, ra[c]);
      tmem_ld_wait();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float o0 = __uint_as_float(ra[c][2 * i]) * sc, o1 = __uint_as_float(ra[c][2 * i + 1]) * sc;
          hi[i] = pack_bf16x2(o0, o1);
          lo[i] = pack_bf16x2(o0 - bf16_lo_to_f32(hi[i]), o1 - bf16_hi_to_f32(hi[i]));
        }
        tmem_st16(lane_addr + C::TM_OL + c * 16, hi);
        tmem_st16(lane_addr + C::TM_OL + D / 2 + c * 16, lo);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->a2_full);
      lin_ok = mbar_wait_warp(&sh->y_done, 0, limit_ns);
      if (!lin_ok) ok = false;
      tc_fence_after();
    }
    if (ok) {
      // out = O / l  -> bf16 staging over the K/V tiles -> one TMA store per 64 columns
      const uint32_t st_addr = sbase + C::OFF_K;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t ro[32];
        if (n >= 1 || lin_ok) {
          tmem_ld32(lane_addr + C::TM_O + c * 32, ro);
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ro[i] = 0u;
        }
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          packed[i] = pack_bf16x2(__uint_as_float(ro[2 * i]) * inv_l, __uint_as_float(ro[2 * i + 1]) * inv_l);
        const int ch = (c * 32) / 64, pc0 = ((c * 32) % 64) / 8;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          st_shared_v4(st_addr + ch * 16384 + sw128_offset((uint32_t)r, (uint32_t)(pc0 + k)), packed[4 * k],
                       packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
      }
      fence_proxy_async_smem();
    } else {
      record_timeout(sh, status);
    }
    named_bar_sync(1, 128);
    if (threadIdx.x == 32 && !sh->abort_flag) {
#pragma unroll
      for (int ch = 0; ch < C::DCH; ++ch)
        tma_store_3d(&tm_out, smem + C::OFF_K + ch * 16384, h * D + ch * 64, qtile * 128, b);
      bulk_commit_group();
      bulk_wait_group_read0();
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

template <int D, int BLK>
cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t s) {
  using C = AttnCfg<D, BLK>;
  cudaError_t e =
      cudaFuncSetAttribute(salad_attn_kernel<D, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(salad_attn_kernel<D, BLK>, cudaFuncAttributePreferredSharedMemoryCarveout,
                           cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  const int qtiles = (a.N + 127) / 128;
  const long long grid = (long long)qtiles * a.B * a.heads;
  salad_attn_kernel<D, BLK><<<(unsigned)grid, 160, C::SMEM, s>>>(
      *a.tm_q, *a.tm_k, *a.tm_v, *a.tm_out, *a.tm_sz, *a.tm_w, a.row_ptr, a.col_idx, a.gate, a.sz, a.heads, a.N,
      qtiles, a.scale_log2, a.eps, a.status, a.wait_limit_ns);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  if (a.d == 64) return a.block == 64 ? launch_attn_t<64, 64>(a, s) : launch_attn_t<64, 128>(a, s);
  return a.block == 64 ? launch_attn_t<128, 64>(a, s) : launch_attn_t<128, 128>(a, s);
}

}  // namespace salad
