// Linear-branch state of SALAD's ReLU linear attention (SALAD summary section
// 2.1: a ReLU-based linear attention of O(N) cost that carries global token
// interactions).  Per (b, h), over all N tokens:
//   S[c][e] = sum_j relu(k_j[c]) v_j[e]        z[c] = sum_j relu(k_j[c])
//
// linear_partial_kernel: grid (splits, B*Hh).  Each CTA streams its share of
// 64-token chunks through a 3-stage TMA ring; four warps apply ReLU to the K
// tile in shared memory (accumulating z in fp32 on the way) and one thread
// issues tcgen05 MMAs  D[c][e] += relu(K)^T[c][tok] * V[tok][e]  with both
// operands MN-major and the fp32 accumulator in tensor memory.  The CTA writes
// its partial S and z in fp32.
// linear_finalize_kernel: fixed-order sum of the partials (deterministic), then
// z in fp32 with S in fp32 (the state export), the projected state S W as bf16
// hi + lo halves in the B operand layout the attention epilogue feeds to the
// tensor cores (the forward), or both (the layer backward).
#include "internal.h"
#include "ptx.cuh"

#include <cuda_bf16.h>

namespace salad {
namespace {

constexpr int kTok = 64;      // tokens per chunk
constexpr int kStages = 3;
constexpr uint64_t kDrainNs = 1000000000ull;

struct LinShared {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t relu[kStages];
  uint64_t acc_done;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
  float zred[256];
};

template <int D>
struct LinCfg {
  static constexpr int BOX_BYTES = kTok * 128;          // one [64 tokens x 64 cols] bf16 box
  static constexpr int TILE_BYTES = (D / 64) * BOX_BYTES;
  static constexpr int STAGE_BYTES = 2 * TILE_BYTES;    // K tile then V tile
  static constexpr int OFF_BAR = kStages * STAGE_BYTES;
  static constexpr int SMEM = OFF_BAR + (int)sizeof(LinShared) + 1024;  // + alignment slack
  // M is padded to 128 for D = 64: the second 64-row half of A reads the V tile
  // and lands in accumulator rows 64..127, which are never read.
  static constexpr uint32_t IDESC = idesc_bf16(128, D, true, true);
};



__device__ __forceinline__ void record_timeout(LinShared* sh, uint32_t* status) {
  sh->abort_flag = 1;
  atomicOr(status, kStatusTimeout);
}

template <int D>
__global__ void __launch_bounds__(192, 1)
    linear_partial_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                          const float* __restrict__ gate, float* __restrict__ partial, int heads, int N,
                          int chunks_per_split, uint32_t* work_ctr, uint32_t* status, uint64_t limit_ns) {
  using C = LinCfg<D>;
  const int split = blockIdx.x, bh = blockIdx.y, BH = gridDim.y;
  // the attention kernel that follows in the stream hands out its work items from this counter
  if (split == 0 && bh == 0 && threadIdx.x == 0) *work_ctr = 0u;
  if (gate != nullptr && gate[bh] == 0.0f) return;  // branch dropped for this (b, h)
  const int b = bh / heads, h = bh % heads;
  const int total_chunks = (N + kTok - 1) / kTok;
  const int c_begin = split * chunks_per_split;
  const int n_chunks = min(total_chunks, c_begin + chunks_per_split) - c_begin;  // >= 1 by construction

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  LinShared* sh = reinterpret_cast<LinShared*>(smem + C::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
      mbar_init(&sh->relu[s], 4);
    }
    mbar_init(&sh->acc_done, 1);
    mbar_init(&sh->drain, 1);
    sh->abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_map(&tm_k);
    tma_prefetch_map(&tm_v);
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int issued = 0;
      for (int it = 0; it < n_chunks; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (sh->abort_flag || !mbar_wait(&sh->empty[s], ph ^ 1, limit_ns)) {
          record_timeout(sh, status);
          break;
        }
        uint8_t* kt = smem + s * C::STAGE_BYTES;
        uint8_t* vt = kt + C::TILE_BYTES;
        mbar_arrive_expect_tx(&sh->full[s], C::STAGE_BYTES);
        const int row = (c_begin + it) * kTok;
#pragma unroll
        for (int ch = 0; ch < D / 64; ++ch) {
          tma_load_3d(kt + ch * C::BOX_BYTES, &tm_k, &sh->full[s], h * D + ch * 64, row, b);
          tma_load_3d(vt + ch * C::BOX_BYTES, &tm_v, &sh->full[s], h * D + ch * 64, row, b);
        }
        issued = it + 1;
      }
      if (sh->abort_flag) {
        // let every copy this thread started land before the CTA can exit
        for (int it = (issued > kStages ? issued - kStages : 0); it < issued; ++it)
          mbar_wait(&sh->full[it % kStages], (it / kStages) & 1, kDrainNs);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      for (int it = 0; it < n_chunks; ++it) {
        const int s = it % kStages;
        const uint32_t ph = (it / kStages) & 1;
        if (sh->abort_flag || !mbar_wait(&sh->relu[s], ph, limit_ns)) {
          record_timeout(sh, status);
          break;
        }
        tc_fence_after();
        const uint32_t kt = smem_u32(smem + s * C::STAGE_BYTES);
        const uint32_t vt = kt + C::TILE_BYTES;
#pragma unroll
        for (int kk = 0; kk < kTok / 16; ++kk) {
          const uint64_t a = sw128_desc(kt + kk * 2048, C::BOX_BYTES, 1024);
          const uint64_t bdesc = sw128_desc(vt + kk * 2048, C::BOX_BYTES, 1024);
          mma_bf16_ss(tmem, a, bdesc, C::IDESC, (it > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sh->empty[s]);
      }
      if (sh->abort_flag) {
        mma_commit(&sh->drain);
        mbar_wait(&sh->drain, 0, kDrainNs);
      } else {
        mma_commit(&sh->acc_done);
      }
    }
  } else {
    // ---------------- ReLU + z (warps 2..5), then the accumulator write-out
    const int t = threadIdx.x - 64;           // 0..127
    constexpr int PAIRS = D / 2;               // bf16 pairs per token row
    constexpr int RSTEP = 128 / PAIRS;         // threads sharing a column pair
    const int p = t % PAIRS, r0 = t / PAIRS;
    const uint32_t col_off = (uint32_t)(p / 32) * C::BOX_BYTES;
    const uint32_t piece = (uint32_t)((p % 32) / 4), word = (uint32_t)(p % 4) * 4;
    float z0 = 0.f, z1 = 0.f;
    bool ok = true;
    for (int it = 0; it < n_chunks && ok; ++it) {
      const int s = it % kStages;
      const uint32_t ph = (it / kStages) & 1;
      if (sh->abort_flag || !mbar_wait(&sh->full[s], ph, limit_ns)) {
        record_timeout(sh, status);
        ok = false;
        break;
      }
      const uint32_t kt = smem_u32(smem + s * C::STAGE_BYTES) + col_off;
      // the rows of this column pair in batches: all loads of a batch, then its
      // stores (one shared-memory round trip per batch, not per row)
      constexpr int NR = kTok / RSTEP, BATCH = NR < 16 ? NR : 16;
#pragma unroll
      for (int r1 = 0; r1 < NR; r1 += BATCH) {
        uint32_t v[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const uint32_t addr = kt + sw128_offset((uint32_t)(r0 + (r1 + i) * RSTEP), piece) + word;
          asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v[i]) : "r"(addr));
        }
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          const uint32_t neg = ((v[i] >> 15) & 0x00010001u) * 0xFFFFu;  // 0xFFFF in each negative half
          v[i] &= ~neg;
          const uint32_t addr = kt + sw128_offset((uint32_t)(r0 + (r1 + i) * RSTEP), piece) + word;
          asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v[i]) : "memory");
        }
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
          z0 += bf16_lo_to_f32(v[i]);
          z1 += bf16_hi_to_f32(v[i]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->relu[s]);
    }
    // z: fixed-order reduction of the threads that share a column pair
    sh->zred[2 * t] = z0;
    sh->zred[2 * t + 1] = z1;
    named_bar_sync(1, 128);
    float* dst = partial + ((size_t)split * BH + bh) * (size_t)(D + 1) * D;
    if (t < D) {
      float zc = 0.f;
      for (int k = 0; k < RSTEP; ++k) zc += sh->zred[2 * ((t / 2) + k * PAIRS) + (t & 1)];
      dst[(size_t)D * D + t] = zc;
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && mbar_wait_warp(&sh->acc_done, 0, limit_ns)) {
      tc_fence_after();
      const int quarter = warp & 3;
      const int c = quarter * 32 + lane;  // accumulator row = feature c of relu(k)
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + cc * 32, r);
        tmem_ld_wait();
        if (c < D) {
          float4* row = reinterpret_cast<float4*>(dst + (size_t)c * D + cc * 32);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            row[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                                 __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
        }
      }
    } else if (ok) {
      record_timeout(sh, status);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// grid (B*Hh, D/ROWS), 256 threads.  CTA (bh, g) owns features c in
// [ROWS*g, ROWS*g + ROWS): it sums their split partials in split order (float4
// loads, coalesced along e), a fixed order, so results do not vary run to run,
// and writes z_out[bh][c] in fp32 and
//   WRITE_S: S_out[bh][c][e] in fp32 (salad_linear_state, the layer backward).
//   WRITE_T: the projected state T = S W,
//            T[c][f] = sum_e S[c][e] W[e][f], transposed and split into bf16
//            hi + lo halves: t_op[bh][f][c] = hi(T[c][f]), t_op[bh][f][D+c] =
//            lo(T[c][f]).  That is the K-major B operand of the attention
//            epilogue's U = relu(q) T, so the projection is applied to the state
//            once per (b, h) instead of to every query row:
//            (relu(q) S / den) W = relu(q) (S W) / den.
template <int D, bool WRITE_S, bool WRITE_T>
__global__ void __launch_bounds__(256) linear_finalize_kernel(const float* __restrict__ partial,
                                                              const float* __restrict__ gate,
                                                              const uint16_t* __restrict__ w,
                                                              uint16_t* __restrict__ t_op, float* __restrict__ z_out,
                                                              float* __restrict__ S_out, int splits) {
  constexpr int E4 = D / 4;        // float4 per partial row
  constexpr int ROWS = 256 / E4;   // features per CTA: 8 (d = 128) or 16 (d = 64)
  constexpr int FG = 256 / D;      // thread groups sharing a projected column f
  constexpr int RPT = ROWS / FG;   // rows of T per thread: 4
  constexpr int WV = D * D / 8;    // 16-byte pieces of W
  const int bh = blockIdx.x, g = blockIdx.y, BH = gridDim.x;
  if (gate != nullptr && gate[bh] == 0.0f) return;
  __shared__ __align__(16) float acc[ROWS][D];
  __shared__ __align__(16) uint16_t wsm[WRITE_T ? D * D : 8];
  const int t = threadIdx.x, rr = t / E4, e4 = (t % E4) * 4;
  if constexpr (WRITE_T) {
    // W into shared memory first: its loads are in flight with the partials'
    uint4 wv[WV / 256];
#pragma unroll
    for (int i = 0; i < WV / 256; ++i) wv[i] = __ldg(reinterpret_cast<const uint4*>(w) + i * 256 + t);
#pragma unroll
    for (int i = 0; i < WV / 256; ++i) reinterpret_cast<uint4*>(wsm)[i * 256 + t] = wv[i];
  }
  const size_t slab = (size_t)(D + 1) * D, split_stride = (size_t)BH * slab;
  const float4* src = reinterpret_cast<const float4*>(partial + (size_t)bh * slab + (size_t)(ROWS * g + rr) * D + e4);
  const size_t step4 = split_stride / 4;
  float4 s = make_float4(0.f, 0.f, 0.f, 0.f);
  int sp = 0;
  for (; sp + 8 <= splits; sp += 8) {
    float4 a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = src[(size_t)(sp + i) * step4];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      s.x += a[i].x;
      s.y += a[i].y;
      s.z += a[i].z;
      s.w += a[i].w;
    }
  }
  for (; sp < splits; ++sp) {
    const float4 a0 = src[(size_t)sp * step4];
    s.x += a0.x;
    s.y += a0.y;
    s.z += a0.z;
    s.w += a0.w;
  }
  if (t < ROWS) {
    const float* zsrc = partial + (size_t)bh * slab + (size_t)D * D + ROWS * g + t;
    // eight independent loads at a time, added in split order
    float z = 0.f;
    int q = 0;
    for (; q + 8 <= splits; q += 8) {
      float a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = zsrc[(size_t)(q + i) * split_stride];
#pragma unroll
      for (int i = 0; i < 8; ++i) z += a[i];
    }
    for (; q < splits; ++q) z += zsrc[(size_t)q * split_stride];
    z_out[(size_t)bh * D + ROWS * g + t] = z;
  }
  if constexpr (WRITE_S) {
    float* dst = S_out + ((size_t)bh * D + ROWS * g + rr) * D + e4;  // S_out is only 4-byte aligned
    dst[0] = s.x;
    dst[1] = s.y;
    dst[2] = s.z;
    dst[3] = s.w;
  }
  if constexpr (WRITE_T) {
    *reinterpret_cast<float4*>(&acc[rr][e4]) = s;
    __syncthreads();
    // thread (f, fg): T rows ROWS*g + fg*RPT + k, column f
    const int f = t % D, fg = t / D;
    float tr[RPT];
#pragma unroll
    for (int k = 0; k < RPT; ++k) tr[k] = 0.f;
#pragma unroll 4
    for (int e = 0; e < D; e += 4) {
      float we[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) we[i] = __uint_as_float((uint32_t)wsm[(e + i) * D + f] << 16);
#pragma unroll
      for (int k = 0; k < RPT; ++k) {
        const float4 sv = *reinterpret_cast<const float4*>(&acc[fg * RPT + k][e]);
        tr[k] = fmaf(sv.x, we[0], tr[k]);
        tr[k] = fmaf(sv.y, we[1], tr[k]);
        tr[k] = fmaf(sv.z, we[2], tr[k]);
        tr[k] = fmaf(sv.w, we[3], tr[k]);
      }
    }
    uint32_t hi[RPT / 2], lo[RPT / 2];
#pragma unroll
    for (int k = 0; k < RPT; k += 2) {
      const uint32_t h = pack_bf16x2(tr[k], tr[k + 1]);
      hi[k / 2] = h;
      lo[k / 2] = pack_bf16x2(tr[k] - bf16_lo_to_f32(h), tr[k + 1] - bf16_hi_to_f32(h));
    }
    uint16_t* row = t_op + ((size_t)bh * D + f) * (2 * D) + ROWS * g + fg * RPT;
    *reinterpret_cast<uint2*>(row) = make_uint2(hi[0], hi[1]);
    *reinterpret_cast<uint2*>(row + D) = make_uint2(lo[0], lo[1]);
  }
}

template <int D>
cudaError_t launch_linear_t(const LinearArgs& a, cudaStream_t s) {
  using C = LinCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(linear_partial_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM);
  if (e != cudaSuccess) return e;
  const int BH = a.B * a.heads;
  linear_partial_kernel<D><<<dim3(a.splits, BH), 192, C::SMEM, s>>>(
      *a.tm_k, *a.tm_v, a.gate, a.partial, a.heads, a.N, a.chunks_per_split, a.work_ctr, a.status,
      a.wait_limit_ns);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 fgrid(BH, D / (256 / (D / 4)));
  if (a.S_out != nullptr && a.with_t)
    linear_finalize_kernel<D, true, true><<<fgrid, 256, 0, s>>>(a.partial, a.gate, a.w, a.t_op, a.z, a.S_out,
                                                               a.splits);
  else if (a.S_out != nullptr)
    linear_finalize_kernel<D, true, false><<<fgrid, 256, 0, s>>>(a.partial, a.gate, nullptr, nullptr, a.z,
                                                                a.S_out, a.splits);
  else
    linear_finalize_kernel<D, false, true><<<fgrid, 256, 0, s>>>(a.partial, a.gate, a.w, a.t_op, a.z, nullptr,
                                                                a.splits);
  return cudaGetLastError();
}

}  // namespace

WorkspaceLayout workspace_layout(int B, int N, int heads, int d) {
  WorkspaceLayout L{};
  const long long BH = (long long)B * heads;
  const int total_chunks = (N + kTok - 1) / kTok;
  // about two CTAs per SM of a 148-SM B200 in one wave
  int splits = (int)(296 / BH);
  if (splits < 1) splits = 1;
  if (splits > total_chunks) splits = total_chunks;
  const int cps = (total_chunks + splits - 1) / splits;
  splits = (total_chunks + cps - 1) / cps;  // every split owns at least one chunk
  L.splits = splits;
  L.chunks_per_split = cps;
  auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
  L.off_status = 0;
  L.off_t = 256;
  L.off_z = L.off_t + up((size_t)BH * d * (2 * d) * 2);
  L.off_partial = L.off_z + up((size_t)BH * d * 4);
  L.total = L.off_partial + up((size_t)splits * BH * (d + 1) * d * 4);
  return L;
}

cudaError_t launch_linear_reduce(const LinearArgs& a, cudaStream_t s) {
  return a.d == 64 ? launch_linear_t<64>(a, s) : launch_linear_t<128>(a, s);
}

}  // namespace salad
