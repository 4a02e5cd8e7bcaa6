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
// topk_pool_kernel    grid (nb, B*Hh), D threads: thread t < D/2 the means of q
//                     for features 2t and 2t+1 (4-byte loads, each feature's sum
//                     still in token order), thread D/2 + t those of k; CTA
//                     (I, bh) also writes row_ptr (every row has K entries).
// topk_select_kernel  grid (B*Hh, ceil(nb / 8)), 256 threads: the scores of 8
//                     query blocks against every key block (chunks of 64 key
//                     means staged in shared memory, two chains per thread),
//                     then one warp per query block takes the K best
//                     key blocks in K rounds of a warp-wide maximum over
//                     (score, then the smaller J) and writes them in order.
// Memory: the pooling reads q and k once (4*d bytes per token per (b, h)); the
// scores are nb^2 * d fused multiply-adds per (b, h).
#include "internal.h"

namespace salad {
namespace {

constexpr int kRows = 8;        // query blocks per selection CTA (one per warp)
constexpr int kChunk = 64;      // key blocks staged at a time
constexpr int kKeysInRegs = 8;  // rank keys a lane keeps in registers (rows of up to 256 key blocks)

template <int D>
__global__ void __launch_bounds__(D) topk_pool_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ k,
                                                      int N, int heads, int blk, int nb, int kk,
                                                      float* __restrict__ qm, float* __restrict__ km,
                                                      int32_t* __restrict__ row_ptr) {
  const int I = blockIdx.x, bh = blockIdx.y, b = bh / heads, h = bh % heads;
  const int t = threadIdx.x;
  const bool is_k = t >= D / 2;
  const int c = 2 * (is_k ? t - D / 2 : t);  // features c and c + 1
  const uint32_t* src = reinterpret_cast<const uint32_t*>(is_k ? k : q);
  const int t0 = I * blk, t1 = min(N, t0 + blk);
  float s0 = 0.f, s1 = 0.f;
#pragma unroll 16
  for (int tok = t0; tok < t1; ++tok) {
    const uint32_t x = src[((((size_t)b * N + tok) * heads + h) * D + c) / 2];
    s0 += __uint_as_float(x << 16);
    s1 += __uint_as_float(x & 0xFFFF0000u);
  }
  float* dst = (is_k ? km : qm) + ((size_t)bh * nb + I) * D + c;
  dst[0] = s0 / (float)(t1 - t0);
  dst[1] = s1 / (float)(t1 - t0);
  if (t == 0) {
    const long long r = (long long)bh * nb + I;
    row_ptr[r] = (int32_t)(r * kk);
    if (r == (long long)gridDim.y * nb - 1) row_ptr[r + 1] = (int32_t)((r + 1) * kk);
  }
}

// The rank key of a score: larger for a higher score, then for a smaller J
// (-0 ranks with +0, as the float comparison does).
__device__ __forceinline__ uint64_t rank_key(float score, int J) {
  uint32_t u = __float_as_uint(score);
  if (u == 0x80000000u) u = 0u;
  const uint32_t ord = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending with the float
  return ((uint64_t)ord << 32) | (uint32_t)(~(uint32_t)J);
}

__device__ __forceinline__ uint64_t warp_max_u64(uint64_t m) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const uint64_t other = __shfl_xor_sync(0xffffffffu, m, o);
    m = other > m ? other : m;
  }
  return m;
}

template <int D>
__global__ void __launch_bounds__(256) topk_select_kernel(const float* __restrict__ qm, const float* __restrict__ km,
                                                          int nb, int kk, int32_t* __restrict__ col_idx) {
  extern __shared__ float tk_smem[];
  constexpr int LD = D + 1;  // padded rows: the key-block rows a warp reads sit in different banks
  float* qs = tk_smem;                       // [kRows][LD]
  float* ks = qs + kRows * LD;               // [kChunk][LD]
  float* sc = ks + kChunk * LD;              // [kRows][nb]
  uint8_t* keep_flag = reinterpret_cast<uint8_t*>(sc + kRows * nb);  // [kRows][nb]
  const int bh = blockIdx.x, I0 = blockIdx.y * kRows, tid = threadIdx.x;
  const int nr = min(kRows, nb - I0);
  for (int x = tid; x < nr * D; x += 256) qs[(x / D) * LD + x % D] = qm[((size_t)bh * nb + I0) * D + x];
  // thread (i, jq): query block I0 + i against key blocks J0 + jq and J0 + jq + 32
  // (two independent chains, each in feature order)
  const int i = tid / 32, jq = tid % 32;
  for (int J0 = 0; J0 < nb; J0 += kChunk) {
    const int nj = min(kChunk, nb - J0);
    __syncthreads();
    for (int x = tid; x < nj * D; x += 256) ks[(x / D) * LD + x % D] = km[((size_t)bh * nb + J0) * D + x];
    __syncthreads();
    if (i < nr) {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll 8
      for (int c = 0; c < D; ++c) {
        const float qv = qs[i * LD + c];
        a0 = fmaf(qv, ks[jq * LD + c], a0);
        a1 = fmaf(qv, ks[(jq + 32) * LD + c], a1);
      }
      if (jq < nj) sc[i * nb + J0 + jq] = a0;
      if (jq + 32 < nj) sc[i * nb + J0 + jq + 32] = a1;
    }
  }
  __syncthreads();
  // one warp per query block: kk rounds of a warp-wide maximum of the rank keys;
  // lane l holds the key blocks J = l, l + 32, ...
  const int warp = tid >> 5, lane = tid & 31;
  if (warp < nr) {
    const float* srow = sc + warp * nb;
    uint8_t* flags = keep_flag + warp * nb;
    for (int J = lane; J < nb; J += 32) flags[J] = kk >= nb ? 1 : 0;
    if (kk < nb) {
      if (nb <= 32 * kKeysInRegs) {
        uint64_t key[kKeysInRegs];
#pragma unroll
        for (int t = 0; t < kKeysInRegs; ++t) {
          const int J = lane + 32 * t;
          key[t] = J < nb ? rank_key(srow[J], J) : 0ull;  // 0: below every real key
        }
        for (int round = 0; round < kk; ++round) {
          uint64_t best = 0;
          int best_t = 0;
#pragma unroll
          for (int t = 0; t < kKeysInRegs; ++t)
            if (key[t] > best) {
              best = key[t];
              best_t = t;
            }
          const uint64_t m = warp_max_u64(best);  // every lane takes part in the shuffles
          if (best != 0 && best == m) {           // keys are unique: one lane wins
            flags[lane + 32 * best_t] = 1;
#pragma unroll
            for (int t = 0; t < kKeysInRegs; ++t)
              if (t == best_t) key[t] = 0;
          }
        }
      } else {
        const int per_lane = (nb + 31) / 32;  // <= 64
        uint64_t taken = 0;
        for (int round = 0; round < kk; ++round) {
          uint64_t best = 0;
          int best_t = -1;
          for (int t = 0; t < per_lane; ++t) {
            const int J = lane + 32 * t;
            if (J < nb && !((taken >> t) & 1ull)) {
              const uint64_t kv = rank_key(srow[J], J);
              if (kv > best) {
                best = kv;
                best_t = t;
              }
            }
          }
          const uint64_t m = warp_max_u64(best);  // every lane takes part in the shuffles
          if (best_t >= 0 && best == m) {
            taken |= 1ull << best_t;
            flags[lane + 32 * best_t] = 1;
          }
        }
      }
    }
    __syncwarp();
    // the kept key blocks in ascending order
    int32_t* out = col_idx + ((size_t)bh * nb + I0 + warp) * kk;
    int base = 0;
    for (int J0 = 0; J0 < nb; J0 += 32) {
      const int J = J0 + lane;
      const bool kept = J < nb && flags[J] != 0;
      const unsigned bal = __ballot_sync(0xffffffffu, kept);
      if (kept) out[base + __popc(bal & ((1u << lane) - 1u))] = J;
      base += __popc(bal);
    }
  }
}

template <int D>
cudaError_t launch_topk_t(const TopkArgs& a, cudaStream_t s) {
  const int BH = a.B * a.heads;
  topk_pool_kernel<D><<<dim3(a.nb, BH), D, 0, s>>>(a.q, a.k, a.N, a.heads, a.block, a.nb, a.kk, a.qm, a.km,
                                                   a.row_ptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem =
      sizeof(float) * (size_t)(kRows * (D + 1) + kChunk * (D + 1) + kRows * a.nb) + kRows * (size_t)a.nb;
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
