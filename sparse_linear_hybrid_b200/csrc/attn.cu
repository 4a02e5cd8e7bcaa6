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
// Work item: one 128-row query tile of one (b, h) (two 64-token query blocks
// when block == 64, whose kept-key lists are merged; a key tile then carries a
// bit per half saying which rows may see it).  The kernel is persistent: one
// CTA per SM takes items from a global counter, so the next item's Q load, K
// loads and first S product run while the softmax warps finish the current
// item.  Every ring below keeps its protocol across items (its index counts
// across the whole CTA).  Warp roles, 384 threads:
//   warp 0     leader and TMA producer: takes the next item (atomic counter,
//              decoded once and handed to the other roles through a 2-slot
//              queue), loads its Q into one of two Q buffers and its K tiles
//              into a 2-deep ring;
//   warp 10    TMA producer of the V tiles (2-deep ring) and of T.  Where T
//              has no region of its own, T_hi goes through the K ring (loaded
//              by warp 0 after the item's last K tile) and T_lo through the V
//              ring (after the item's last V tile);
//   warp 11    output store: one TMA store per item once the softmax warps
//              have staged its tile, then frees that Q buffer;
//   warp 1     tcgen05 issuer (one thread) and TMEM owner: copies the item's Q
//              into tensor memory, S = Q K_j^T into one of two TMEM S buffers
//              (A from tensor memory, K from shared memory); O += P_j V_j with
//              P_j read from TMEM; U = relu(Q) [T_hi ; T_lo] of an item into the
//              S buffer of the slot that follows its tiles, right after its
//              last PV (the next item's Q copy and first S follow U);
//   warps 2-9  softmax, two threads per query row (each takes half of the key
//              columns of a tile and half of the feature columns of O): online
//              softmax whose running maximum is only moved (and O rescaled in
//              TMEM) when it grows by more than 2^8, P_j written to TMEM as
//              bf16; after an item's last tile each thread writes ReLU of its
//              half of its row of Q over the Q columns (the A operand of U) and
//              sums its half of relu(q) . z; finally out = O / l + g U / den is
//              staged in the item's Q buffer for the store warp.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O [256,256+d),
// P [384,384+BLK/2), Q [448,448+d/2) (bf16 pairs).  With Q in tensor memory the
// S products read only K from shared memory.  P_{j+1} is written once PV_j has
// completed (the softmax of tile j+1 outlasts it).  T is fed as a hi + lo pair of
// bf16 halves (K doubled, relu(Q) read twice), so U keeps ~16 mantissa bits of
// T.  Every barrier wait is bounded; on a time-out a role records it, stops and
// drains what it issued.
#include "internal.h"
#include "ptx.cuh"

namespace salad {
namespace {

constexpr uint64_t kDrainNs = 1000000000ull;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: rescale O only when the max grows by > 2^8
constexpr int kThreads = 384;

// Phase stamps of the profiling build (-DSALAD_PROFILE, off by default): four
// recording threads per CTA -- the leader, the tcgen05 issuer, the V producer
// and the first thread of softmax warp 2 -- write (event code << 56 | clock64)
// into their own run of kProfEvents words of a buffer the host hands over
// (salad_profile_set_buffer); sparse_linear_hybrid_b200/profile_phases.py turns
// them into cycles per phase.  The normal build compiles none of it.
#ifdef SALAD_PROFILE
constexpr int kProfEvents = 8192;
constexpr int kProfRecorders = 4;
__device__ uint64_t* g_prof_buf = nullptr;
__device__ int g_prof_ctas = 0;  // CTAs the buffer has room for
#define SALAD_PROF(code)                                                                           \
  do {                                                                                             \
    if (prof_ != nullptr && prof_n_ < kProfEvents)                                                 \
      prof_[prof_n_++] = ((uint64_t)(code) << 56) | ((uint64_t)clock64() & 0x00FFFFFFFFFFFFFFull); \
  } while (0)
#else
#define SALAD_PROF(code) \
  do {                   \
  } while (0)
#endif
// event codes
enum : int {
  kPfLdItem = 1, kPfLdKWait = 2, kPfLdKGot = 3,
  kPfSWait = 10, kPfSReady = 11, kPfSIssued = 12, kPfQCopied = 13, kPfUWait = 14, kPfUIssued = 15,
  kPfPvWait = 20, kPfPvP = 21, kPfPvV = 22, kPfPvIssued = 23,
  kPfVWait = 30, kPfVGot = 31,
  kPfSmWait = 40, kPfSmS = 41, kPfSmLoaded = 42, kPfSmMax = 43, kPfSmXchg = 44, kPfSmExp = 45, kPfSmPv = 46,
  kPfSmP = 47, kPfEpBegin = 50, kPfEpRelu = 51, kPfEpSums = 52, kPfEpU = 53, kPfEpEnd = 54,
};

// A work item as the leader hands it to the other roles (through shared
// memory, so that no other role reads the mask or the gate from global memory
// on its way into an item).
struct Item {
  int w;                // work index; -1: no work left
  int bh, qtile, b, h;
  int n;                // kept key tiles
  int vlast;            // real keys in the last kept tile (BLK unless it is the partial last block)
  int ra, na, rb, nb;   // col_idx ranges of the tile's query block(s) (the second one when BLK == 64)
  float g;              // gate of this (b, h)
  bool lin;             // the linear branch is dropped for this (b, h) when its gate is 0
};

struct AttnShared {
  uint64_t item_full[2], item_empty[2];  // the 2-slot item queue
  uint64_t q_full[2], q_free[2], q_relu[2], staged[2];  // per Q buffer
  uint64_t k_full[2], k_empty[2], v_full[2], v_empty[2];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], pv_done[2];
  uint64_t t_full, t_empty;
  uint64_t z_full[2];        // per item slot: z of the item's (b, h) has landed in zs
  uint64_t drain;
  uint64_t xbar[4];          // per lane quarter: the two halves of its rows meet here (64 arrivals)
  Item item[2];
  uint32_t tmem_base;
  volatile int abort_flag;
  float xmax[2][2][128];     // per exchange parity, per half: partial row maxima
  float xsum[2][2][128];     // per exchange parity, per half: partial row sums
  float xlse[2][2][128];     // the same of the unrounded p (log-sum-exp output)
  float xden[2][2][128];     // per exchange parity, per half: partial relu(q) . z
  alignas(16) float zs[2][128];  // per item slot: z of the item's (b, h)
  int k_edge[2];             // tile blocks: per K ring stage, which grid edges its box sticks out of
};

template <int D, int BLK>
struct AttnCfg {
  static constexpr int QROWS = 128;
  static constexpr int DCH = D / 64;                // 64-column chunks of a d-wide row
  static constexpr int Q_BYTES = QROWS * D * 2;     // DCH chunks of 16 KB
  static constexpr int KV_BOX = BLK * 128;          // one [BLK x 64] box
  static constexpr int KV_BYTES = DCH * KV_BOX;     // one K or V tile
  static constexpr int T_CH = 2 * D / 64;           // 64-column chunks of the [T_hi | T_lo] operand
  static constexpr int T_CH_BYTES = D * 128;        // D rows (feature f) of 128 bytes
  static constexpr int T_BYTES = T_CH * T_CH_BYTES;
  static constexpr int BASE_BYTES = 2 * Q_BYTES + 4 * KV_BYTES;  // Q[2], K[2], V[2]
  // T has a region of its own when shared memory allows.  Otherwise its two
  // halves travel through the rings as one extra entry each, right after the
  // item's last K and V tiles.  Their stages free up while the item's last
  // tile is still in the softmax, so U need not wait for the last PV.
  static constexpr bool T_IN_RINGS = BASE_BYTES + T_BYTES + (int)sizeof(AttnShared) + 1024 > 232448;
  static constexpr int OFF_Q0 = 0;
  static constexpr int OFF_K0 = 2 * Q_BYTES;
  static constexpr int OFF_V0 = OFF_K0 + 2 * KV_BYTES;
  static constexpr int OFF_T = BASE_BYTES;  // dedicated T region (unused when T_IN_RINGS)
  static constexpr int OFF_BAR = BASE_BYTES + (T_IN_RINGS ? 0 : T_BYTES);
  static constexpr int SMEM_USED = OFF_BAR + (int)sizeof(AttnShared) + 1024;
  // at least 120 KB so that one CTA (and its 512 TMEM columns) owns the SM
  static constexpr int SMEM = SMEM_USED > 122880 ? SMEM_USED : 122880;
  // tile blocks: four 128 x 16 bf16 operands in the 32-byte-swizzled K-major
  // layout (4 KB each) -- a tile of ones and the key-padding bias of a box at
  // the right edge, the bottom edge and both -- after the barriers
  static constexpr int MASK_OP_BYTES = 128 * 32;
  static constexpr int OFF_MASK = (OFF_BAR + (int)sizeof(AttnShared) + 1023) / 1024 * 1024;
  static constexpr int SMEM_TILES = OFF_MASK + 4 * MASK_OP_BYTES + 1024;
  static_assert(SMEM_TILES <= 232448, "shared memory budget (tile blocks)");
  static constexpr uint32_t TM_S0 = 0, TM_S1 = 128, TM_O = 256, TM_P = 384, TM_Q = 448;
  static constexpr uint32_t P_COLS = BLK / 2;       // the P buffer: BLK bf16 per row
  static constexpr uint32_t Q_COLS = D / 2;         // Q (then relu(Q)) in tensor memory: D bf16 per row
  static constexpr uint32_t IDESC_S = idesc_bf16(128, BLK, false, false);   // Q K^T
  static constexpr uint32_t IDESC_PV = idesc_bf16(128, D, false, true);     // P V   (V MN-major)
  static constexpr uint32_t IDESC_U = idesc_bf16(128, D, false, false);     // relu(Q) [T_hi ; T_lo]
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(!T_IN_RINGS || (T_BYTES == 2 * KV_BYTES && T_CH == 2 * DCH && T_CH_BYTES == KV_BOX),
                "each half of T must have the layout of one K or V tile");
  static_assert(TM_P + P_COLS <= TM_Q && TM_Q + Q_COLS <= 512 && D <= 128, "tensor memory budget");
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

template <int BLK, bool TILES>
__device__ __forceinline__ Item make_item(int w, int qtiles, int heads, int N, int nb, const int32_t* row_ptr,
                                          const int32_t* col_idx, const float* gate, int mask_per_bh,
                                          int mask_rows, uint32_t* status) {
  Item im;
  im.w = w;
  im.bh = w / qtiles;
  im.qtile = w % qtiles;
  im.b = im.bh / heads;
  im.h = im.bh % heads;
  im.g = gate[im.bh];
  im.lin = im.g != 0.0f;
  // the mask's rows are per head, or per (b, h) for a data-dependent mask
  KeyIter it = make_iter<BLK>(row_ptr, col_idx, mask_per_bh ? im.bh : im.h, nb, im.qtile);
  {
    // debug builds: a malformed row of the item reads as no kept key blocks
    const int r0 = (mask_per_bh ? im.bh : im.h) * nb + (BLK == 128 ? im.qtile : 2 * im.qtile);
    bool ok = debug_row_ok(row_ptr, col_idx, r0, mask_rows, nb, true, status);
    if (BLK != 128 && 2 * im.qtile + 1 < nb) ok = debug_row_ok(row_ptr, col_idx, r0 + 1, mask_rows, nb, true, status) && ok;
    if (!ok) {
      it.a = col_idx;
      it.na = 0;
      it.b = nullptr;
      it.nb = 0;
    }
  }
  im.ra = (int)(it.a - col_idx);
  im.na = it.na;
  im.rb = it.b ? (int)(it.b - col_idx) : 0;
  im.nb = it.nb;
  int last = -1;
  if (BLK == 128) {
    im.n = it.na;
    if (it.na > 0) last = it.a[it.na - 1];
  } else {
    int col, bits, n = 0;
    while (it.next(col, bits)) {
      ++n;
      last = col;
    }
    im.n = n;
  }
  // (a tile block is never cut short along t; its columns outside the grid are
  // masked by position instead)
  im.vlast = (last >= 0 && !TILES) ? min(BLK, N - last * BLK) : BLK;
  return im;
}

// The kept key tiles of a published item, in the order make_iter yields them.
__device__ __forceinline__ KeyIter item_iter(const Item& im, const int32_t* col_idx) {
  KeyIter it{};
  it.a = col_idx + im.ra;
  it.na = im.na;
  it.b = im.nb > 0 ? col_idx + im.rb : nullptr;
  it.nb = im.nb;
  it.ia = it.ib = 0;
  return it;
}

__device__ __forceinline__ void record_timeout(AttnShared* sh, uint32_t* status) {
  sh->abort_flag = 1;
  atomicOr(status, kStatusTimeout);
}

// TMA copies of one block of rows.  Raster blocks: rows [row0, row0 + rows)
// of the (Hh*d, N, B) view.  Tile blocks: box I of the (Hh*d, W, H, B*T) view,
// whose rows in shared memory follow the slot order (tt*bh + yy)*bw + xx; the
// box's points outside the grid read as zeros and are not written back.
template <bool TILES>
__device__ __forceinline__ void load_block(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int row0,
                                           int I, int b, const TileGeom& g) {
  if constexpr (TILES) {
    const int yt = (int)fastdiv((uint32_t)I, g.div_nw), t = (int)fastdiv((uint32_t)yt, g.div_nh);
    tma_load_4d(dst, map, bar, c0, (I - yt * g.nw) * g.bw, (yt - t * g.nh) * g.bh, b * g.T + t * g.bt);
  } else {
    tma_load_3d(dst, map, bar, c0, row0, b);
  }
}

template <bool TILES>
__device__ __forceinline__ void store_block(const CUtensorMap* map, const void* src, int c0, int row0, int I, int b,
                                            const TileGeom& g) {
  if constexpr (TILES) {
    const int yt = (int)fastdiv((uint32_t)I, g.div_nw), t = (int)fastdiv((uint32_t)yt, g.div_nh);
    tma_store_4d(map, src, c0, (I - yt * g.nw) * g.bw, (yt - t * g.nh) * g.bh, b * g.T + t * g.bt);
  } else {
    tma_store_3d(map, src, c0, row0, b);
  }
}

__device__ __forceinline__ uint32_t relu_bf16x2(uint32_t x) {
  uint32_t r;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(0u));
  return r;
}

template <int D, int BLK, bool TILES>
__global__ void __launch_bounds__(kThreads, 1)
    salad_attn_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_out,
                      const __grid_constant__ CUtensorMap tm_t, const int32_t* __restrict__ row_ptr,
                      const int32_t* __restrict__ col_idx, const float* __restrict__ gate,
                      const float* __restrict__ zvec, int heads, int N, int qtiles, int num_items,
                      uint32_t* work_ctr, float scale_log2, float eps, uint32_t* status, uint64_t limit_ns,
                      int mask_per_bh, const TileGeom tg, float* __restrict__ lse_out) {
  using C = AttnCfg<D, BLK>;
  static_assert(!TILES || BLK == 128, "a tile block fills one 128-row query tile");
  const int nblocks = TILES ? qtiles : (N + BLK - 1) / BLK;  // key blocks per mask row
  const int mask_rows = (mask_per_bh ? num_items / qtiles : heads) * nblocks;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  AttnShared* sh = reinterpret_cast<AttnShared*>(smem + C::OFF_BAR);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sh->item_full[s], 1);
      mbar_init(&sh->item_empty[s], 11);  // V producer, MMA issuer, store thread, 8 softmax warps
      mbar_init(&sh->q_full[s], 1);
      mbar_init(&sh->q_free[s], 1);
      mbar_init(&sh->q_relu[s], 8);
      mbar_init(&sh->staged[s], 8);
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
    mbar_init(&sh->t_empty, 1);
    mbar_init(&sh->z_full[0], 1);
    mbar_init(&sh->z_full[1], 1);
    mbar_init(&sh->drain, 1);
    for (int q = 0; q < 4; ++q) mbar_init(&sh->xbar[q], 64);
    sh->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem_base, 512);
    tmem_relinquish();
  }
  if constexpr (TILES) {
    // Keys of a box outside the grid are masked by the tensor cores: S of a box
    // at an edge gets one more K = 16 product, ones (128 x 16) times the box's
    // bias (128 x 16: row n all 0 when slot n holds a key, all -inf when it lies
    // past the edge), which adds -inf to exactly the padded columns and 0 to the
    // rest.  Rows are uniform, so the swizzle does not move any value.
    uint32_t* mo = reinterpret_cast<uint32_t*>(smem + C::OFF_MASK);
    const int wr = tg.W - (tg.nw - 1) * tg.bw, hr = tg.H - (tg.nh - 1) * tg.bh;  // keys of an edge box
    for (int x = threadIdx.x; x < 4 * C::MASK_OP_BYTES / 4; x += kThreads) {
      const int op = x / (C::MASK_OP_BYTES / 4), row = (x % (C::MASK_OP_BYTES / 4)) / 8;
      uint32_t val = 0x3F803F80u;  // bf16 pair (1, 1)
      if (op > 0) {
        const bool past = ((op & 1) && row % tg.bw >= wr) || ((op & 2) && (row / tg.bw) % tg.bh >= hr);
        val = past ? 0xFF80FF80u : 0u;  // (-inf, -inf) or (0, 0)
      }
      mo[x] = val;
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh->tmem_base;
#ifdef SALAD_PROFILE
  uint64_t* prof_ = nullptr;
  int prof_n_ = 0;
  {
    const int rec = warp == 0 ? 0 : warp == 1 ? 1 : warp == 10 ? 2 : warp == 2 ? 3 : -1;
    if (rec >= 0 && lane == 0 && g_prof_buf != nullptr && (int)blockIdx.x < g_prof_ctas)
      prof_ = g_prof_buf + ((size_t)blockIdx.x * kProfRecorders + rec) * kProfEvents;
  }
#endif

  if (warp == 0) {
    // ============================ leader and TMA producer of Q and K
    if (lane == 0) {
      tma_prefetch_map(&tm_q);
      tma_prefetch_map(&tm_k);
      if (C::T_IN_RINGS) tma_prefetch_map(&tm_t);
      bool ok = true;
      int seq = 0, kj = 0;
      // next K ring entry: wait for its stage, expect its bytes
      auto k_stage = [&](int edge) -> uint8_t* {
        const int s = kj & 1;
        SALAD_PROF(kPfLdKWait);
        // the stage is free once the product that read entry kj - 2 is done.  With
        // T in the rings every K entry feeds exactly one S slot use (S or U) in the
        // same order, so that product's own completion barrier tells; otherwise
        // the products release the stages through k_empty
        const bool free_ok = C::T_IN_RINGS
                                 ? (kj < 2 || mbar_wait(&sh->s_full[s], (uint32_t)(((kj - 2) >> 1) & 1), limit_ns))
                                 : mbar_wait(&sh->k_empty[s], ((kj >> 1) & 1) ^ 1, limit_ns);
        if (sh->abort_flag || !free_ok) return nullptr;
        SALAD_PROF(kPfLdKGot);
        if constexpr (TILES) sh->k_edge[s] = edge;  // read by the MMA thread after k_full
        mbar_arrive_expect_tx(&sh->k_full[s], C::KV_BYTES);
        return smem + C::OFF_K0 + s * C::KV_BYTES;
      };
      for (;;) {
        const int slot = seq & 1;
        const uint32_t ph = (uint32_t)((seq >> 1) & 1);
        // hand the next item to the other roles
        if (sh->abort_flag || !mbar_wait(&sh->item_empty[slot], ph ^ 1, limit_ns)) { ok = false; break; }
        const int w = (int)atomicAdd(work_ctr, 1u);
        SALAD_PROF(kPfLdItem);
        Item im;
        if (w < num_items) {
          im = make_item<BLK, TILES>(w, qtiles, heads, N, nblocks, row_ptr, col_idx, gate, mask_per_bh, mask_rows,
                                     status);
        } else {
          im.w = -1;
        }
        sh->item[slot] = im;
        mbar_arrive(&sh->item_full[slot]);
        if (im.w < 0) break;
        // Q buffer `slot` is free once the output of the item two back has been stored from it
        if (!mbar_wait(&sh->q_free[slot], ph ^ 1, limit_ns)) { ok = false; break; }
        mbar_arrive_expect_tx(&sh->q_full[slot], C::Q_BYTES);
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          load_block<TILES>(smem + C::OFF_Q0 + slot * C::Q_BYTES + ch * 16384, &tm_q, &sh->q_full[slot],
                            im.h * D + ch * 64, im.qtile * 128, im.qtile, im.b, tg);
        KeyIter it = item_iter(im, col_idx);
        int col, bits;
        while (it.next(col, bits)) {
          int edge = 0;
          if constexpr (TILES) {
            // bit 0: the box reaches past W; bit 1: past H
            const int yt = (int)fastdiv((uint32_t)col, tg.div_nw);
            const int xi = col - yt * tg.nw, yi = yt - (int)fastdiv((uint32_t)yt, tg.div_nh) * tg.nh;
            edge = ((xi + 1) * tg.bw > tg.W ? 1 : 0) | ((yi + 1) * tg.bh > tg.H ? 2 : 0);
          }
          uint8_t* kt = k_stage(edge);
          if (!kt) { ok = false; break; }
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            load_block<TILES>(kt + ch * C::KV_BOX, &tm_k, &sh->k_full[kj & 1], im.h * D + ch * 64, col * BLK, col,
                              im.b, tg);
          ++kj;
        }
        if (ok && C::T_IN_RINGS && im.lin) {
          // T_hi: one more K ring entry after the item's key tiles, released by U
          uint8_t* dst = k_stage(0);
          if (!dst) {
            ok = false;
          } else {
#pragma unroll
            for (int ch = 0; ch < C::DCH; ++ch)
              tma_load_3d(dst + ch * C::KV_BOX, &tm_t, &sh->k_full[kj & 1], ch * 64, 0, im.bh);
            ++kj;
          }
        }
        if (!ok) break;
        ++seq;
      }
      if (!ok) record_timeout(sh, status);
      // every copy this thread started lands before the CTA may exit (at once
      // unless another role gave up early)
      for (int i = (seq > 2 ? seq - 2 : 0); i <= seq; ++i)
        if (i < seq || !ok) mbar_wait(&sh->q_full[i & 1], (i >> 1) & 1, kDrainNs);
      for (int i = (kj > 2 ? kj - 2 : 0); i < kj; ++i) mbar_wait(&sh->k_full[i & 1], (i >> 1) & 1, kDrainNs);
    }
  } else if (warp == 10) {
    // ============================ TMA producer of V (and T)
    if (lane == 0) {
      tma_prefetch_map(&tm_v);
      tma_prefetch_map(&tm_t);
      bool ok = true;
      int seq = 0, vj = 0, tl = 0, zc = 0;
      // what last occupied each V stage: a V tile (its global tile index; its PV's
      // pv_done frees the stage) or T_lo (U frees it through v_empty, one phase
      // per T_lo entry of the stage)
      // (kept in scalars: a stage number is only known at run time)
      int gtile = 0, tile0 = -1, tile1 = -1, tlo0 = 0, tlo1 = 0;
      bool is_tlo0 = false, is_tlo1 = false;
      auto v_stage_free = [&](int s) -> bool {
        if (sh->abort_flag) return false;
        if (vj < 2) return true;
        if (s ? is_tlo1 : is_tlo0) return mbar_wait(&sh->v_empty[s], (uint32_t)(((s ? tlo1 : tlo0) - 1) & 1), limit_ns);
        const int g = s ? tile1 : tile0;
        return mbar_wait(&sh->pv_done[g & 1], (uint32_t)((g >> 1) & 1), limit_ns);
      };
      for (;;) {
        const int slot = seq & 1;
        if (sh->abort_flag || !mbar_wait(&sh->item_full[slot], (uint32_t)((seq >> 1) & 1), limit_ns)) {
          ok = false;
          break;
        }
        const Item im = sh->item[slot];
        mbar_arrive(&sh->item_empty[slot]);
        if (im.w < 0) break;
        // z of this (b, h) into zs[slot], once the softmax warps are done with the
        // z of the item two back (they arrive on q_relu after reading it)
        if (seq >= 2 && !mbar_wait(&sh->q_relu[slot], (uint32_t)(((seq - 2) >> 1) & 1), limit_ns)) {
          ok = false;
          break;
        }
        if (im.lin) {
          mbar_arrive_expect_tx(&sh->z_full[slot], D * 4);
          bulk_load(sh->zs[slot], zvec + (size_t)im.bh * D, D * 4, &sh->z_full[slot]);
        } else {
          mbar_arrive(&sh->z_full[slot]);
        }
        ++zc;
        KeyIter it = item_iter(im, col_idx);
        int col, bits;
        while (it.next(col, bits)) {
          const int s = vj & 1;
          SALAD_PROF(kPfVWait);
          if (!v_stage_free(s)) { ok = false; break; }
          SALAD_PROF(kPfVGot);
          if (s) {
            is_tlo1 = false;
            tile1 = gtile;
          } else {
            is_tlo0 = false;
            tile0 = gtile;
          }
          ++gtile;
          mbar_arrive_expect_tx(&sh->v_full[s], C::KV_BYTES);
          uint8_t* vt = smem + C::OFF_V0 + s * C::KV_BYTES;
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            load_block<TILES>(vt + ch * C::KV_BOX, &tm_v, &sh->v_full[s], im.h * D + ch * 64, col * BLK, col, im.b,
                              tg);
          ++vj;
        }
        if (!ok) break;
        if (im.lin && C::T_IN_RINGS) {
          // T_lo: one more V ring entry, released by U
          const int s = vj & 1;
          if (!v_stage_free(s)) { ok = false; break; }
          if (s) {
            is_tlo1 = true;
            ++tlo1;
          } else {
            is_tlo0 = true;
            ++tlo0;
          }
          mbar_arrive_expect_tx(&sh->v_full[s], C::KV_BYTES);
          uint8_t* vt = smem + C::OFF_V0 + s * C::KV_BYTES;
#pragma unroll
          for (int ch = 0; ch < C::DCH; ++ch)
            tma_load_3d(vt + ch * C::KV_BOX, &tm_t, &sh->v_full[s], (C::DCH + ch) * 64, 0, im.bh);
          ++vj;
        } else if (im.lin) {
          if (!mbar_wait(&sh->t_empty, (uint32_t)(tl & 1) ^ 1, limit_ns)) { ok = false; break; }
          mbar_arrive_expect_tx(&sh->t_full, C::T_BYTES);
#pragma unroll
          for (int ch = 0; ch < C::T_CH; ++ch)
            tma_load_3d(smem + C::OFF_T + ch * C::T_CH_BYTES, &tm_t, &sh->t_full, ch * 64, 0, im.bh);
          ++tl;
        }
        ++seq;
      }
      if (!ok) record_timeout(sh, status);
      for (int i = (vj > 2 ? vj - 2 : 0); i < vj; ++i) mbar_wait(&sh->v_full[i & 1], (i >> 1) & 1, kDrainNs);
      for (int i = (zc > 2 ? zc - 2 : 0); i < zc; ++i) mbar_wait(&sh->z_full[i & 1], (i >> 1) & 1, kDrainNs);
      if (tl > 0) mbar_wait(&sh->t_full, (uint32_t)((tl - 1) & 1), kDrainNs);
    }
  } else if (warp == 11) {
    // ============================ output store: once all eight softmax warps
    // have staged an item's tile in its Q buffer, one TMA store, then the
    // buffer is free for the item two ahead
    if (lane == 0) {
      tma_prefetch_map(&tm_out);
      bool ok = true;
      int seq = 0;
      for (;;) {
        const int slot = seq & 1;
        const uint32_t ph = (uint32_t)((seq >> 1) & 1);
        if (sh->abort_flag || !mbar_wait(&sh->item_full[slot], ph, limit_ns)) { ok = false; break; }
        const Item im = sh->item[slot];
        mbar_arrive(&sh->item_empty[slot]);
        if (im.w < 0) break;
        if (!mbar_wait(&sh->staged[slot], ph, limit_ns)) { ok = false; break; }
#pragma unroll
        for (int ch = 0; ch < C::DCH; ++ch)
          store_block<TILES>(&tm_out, smem + C::OFF_Q0 + slot * C::Q_BYTES + ch * 16384, im.h * D + ch * 64,
                             im.qtile * 128, im.qtile, im.b, tg);
        bulk_commit_group();
        bulk_wait_group_read0();
        mbar_arrive(&sh->q_free[slot]);
        ++seq;
      }
      if (!ok) record_timeout(sh, status);
    }
  } else if (warp == 1) {
    // ============================ tcgen05 issuer
    if (lane == 0) {
      bool ok = true;
      int seq = 0, kj = 0, sj = 0, tt = 0, vj = 0, tl = 0;
      // S slot reuse: the softmax frees a slot (s_free) before it signals P of the
      // same tile (p_full), so once this thread has seen p_full of the tile that
      // last used a slot, that slot's s_free wait is already satisfied
      int st = 0, pf_seen = -1, slot_tile0 = -1, slot_tile1 = -1;  // S tiles issued, last p_full seen, per slot
      int q_last = -1;  // S slot index of the last product that read the Q columns (S or U)
      // O += P V for global tile `gt` of the item whose V tiles start at V index
      // `gv0` (P from tensor memory; operands waited for here)
      auto issue_pv = [&](int gt, int gv, bool first) -> bool {
        const int s = gt & 1, vs = gv & 1;
        SALAD_PROF(kPfPvWait);
        if (sh->abort_flag || !mbar_wait(&sh->p_full[s], (uint32_t)((gt >> 1) & 1), limit_ns)) return false;
        SALAD_PROF(kPfPvP);
        if (!mbar_wait(&sh->v_full[vs], (uint32_t)((gv >> 1) & 1), limit_ns)) return false;
        SALAD_PROF(kPfPvV);
        pf_seen = gt;
        tc_fence_after();
        const uint32_t vt = sbase + C::OFF_V0 + vs * C::KV_BYTES;
        const uint32_t pt = tmem + C::TM_P;
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk) {
          const uint64_t bd = sw128_desc(vt + kk * 2048, C::KV_BOX, 1024);
          mma_bf16_ts(tmem + C::TM_O, pt + kk * 8, bd, C::IDESC_PV, (!first || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sh->pv_done[s]);  // also frees the V stage
        SALAD_PROF(kPfPvIssued);
        return true;
      };
      // S = Q K^T into the next S slot (K tile kj of the ring; Q from tensor memory)
      auto issue_s = [&]() -> bool {
        const int s = sj & 1, ks = kj & 1;
        SALAD_PROF(kPfSWait);
        if (sh->abort_flag || !mbar_wait(&sh->k_full[ks], (uint32_t)((kj >> 1) & 1), limit_ns)) return false;
        const int prev = s ? slot_tile1 : slot_tile0;
        const bool implied = prev >= 0 && prev <= pf_seen;
        if (sj >= 2 && !implied && !mbar_wait(&sh->s_free[s], (uint32_t)(((sj - 2) >> 1) & 1), limit_ns))
          return false;
        SALAD_PROF(kPfSReady);
        if (s) {
          slot_tile1 = st;
        } else {
          slot_tile0 = st;
        }
        ++st;
        tc_fence_after();
        const uint32_t kt = sbase + C::OFF_K0 + ks * C::KV_BYTES;
        const uint32_t d_s = tmem + (s ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint64_t bd = sw128_desc(kt + (kk / 4) * C::KV_BOX + (kk % 4) * 32, 16, 1024);
          mma_bf16_ts(d_s, tmem + C::TM_Q + kk * 8, bd, C::IDESC_S, kk > 0 ? 1u : 0u);
        }
        if constexpr (TILES) {
          const int edge = sh->k_edge[ks];
          if (edge != 0)
            mma_bf16_ss(d_s, sw32_desc(sbase + C::OFF_MASK),
                        sw32_desc(sbase + C::OFF_MASK + edge * C::MASK_OP_BYTES), C::IDESC_S, 1u);
        }
        mma_commit(&sh->s_full[s]);  // with T in the rings this also frees the K stage
        if (!C::T_IN_RINGS) mma_commit(&sh->k_empty[ks]);
        q_last = sj;
        ++kj;
        ++sj;
        SALAD_PROF(kPfSIssued);
        return true;
      };
      // U = relu(Q) [T_hi ; T_lo] of the item in Q buffer `qb` (K = 2d: relu(Q)
      // is fed twice) into the S slot after its tiles, completion on s_full like
      // a tile; frees T's place.  T is in its own region, or T_hi is the K ring
      // entry after the item's key tiles and T_lo the V ring entry after them.
      auto issue_u = [&](int qb, int qseq) -> bool {
        const int s = sj & 1, ks = kj & 1, vs = vj & 1;
        const bool t_ok = C::T_IN_RINGS
                              ? mbar_wait(&sh->k_full[ks], (uint32_t)((kj >> 1) & 1), limit_ns) &&
                                    mbar_wait(&sh->v_full[vs], (uint32_t)((vj >> 1) & 1), limit_ns)
                              : mbar_wait(&sh->t_full, (uint32_t)(tl & 1), limit_ns);
        if (sh->abort_flag || !t_ok || !mbar_wait(&sh->q_relu[qb], (uint32_t)((qseq >> 1) & 1), limit_ns))
          return false;
        if (sj >= 2 && !mbar_wait(&sh->s_free[s], (uint32_t)(((sj - 2) >> 1) & 1), limit_ns)) return false;
        SALAD_PROF(kPfUWait);
        if (s) {
          slot_tile1 = -1;
        } else {
          slot_tile0 = -1;
        }
        tc_fence_after();
        const uint32_t t_hi = C::T_IN_RINGS ? sbase + C::OFF_K0 + ks * C::KV_BYTES : sbase + C::OFF_T;
        const uint32_t t_lo = C::T_IN_RINGS ? sbase + C::OFF_V0 + vs * C::KV_BYTES : t_hi + (C::T_CH / 2) * C::T_CH_BYTES;
        const uint32_t d_u = tmem + (s ? C::TM_S1 : C::TM_S0);
#pragma unroll
        for (int kk = 0; kk < 2 * D / 16; ++kk) {
          const int qk = kk % (D / 16), ch = kk / 4;  // ch: 64-column chunk of [T_hi | T_lo]
          const uint32_t tc = ch < C::T_CH / 2 ? t_hi + ch * C::T_CH_BYTES : t_lo + (ch - C::T_CH / 2) * C::T_CH_BYTES;
          const uint64_t bd = sw128_desc(tc + (kk % 4) * 32, 16, 1024);
          mma_bf16_ts(d_u, tmem + C::TM_Q + qk * 8, bd, C::IDESC_U, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sh->s_full[s]);
        if (C::T_IN_RINGS) {
          mma_commit(&sh->v_empty[vs]);  // T_lo's stage (T_hi's K stage is freed through s_full)
          ++kj;
          ++vj;
        } else {
          mma_commit(&sh->t_empty);
          ++tl;
        }
        q_last = sj;
        ++sj;
        SALAD_PROF(kPfUIssued);
        return true;
      };
      for (;;) {
        const int slot = seq & 1;
        if (sh->abort_flag || !mbar_wait(&sh->item_full[slot], (uint32_t)((seq >> 1) & 1), limit_ns)) {
          ok = false;
          break;
        }
        const Item im = sh->item[slot];
        mbar_arrive(&sh->item_empty[slot]);
        if (im.w < 0) break;
        if (!mbar_wait(&sh->q_full[slot], (uint32_t)((seq >> 1) & 1), limit_ns)) { ok = false; break; }
        const uint32_t q_addr = sbase + C::OFF_Q0 + slot * C::Q_BYTES;
        const int n = im.n;
        const int tt0 = tt, vj0 = vj;
        // Q into tensor memory (once the previous item's last S or U has read the
        // columns), then S_0,
        // S_j and PV_{j-1}, ..., PV_{n-1}, then U.  An item without key tiles keeps
        // the Q columns for the relu(Q) its softmax warps write.
        if (n >= 1) {
          // the last product that read the Q columns has completed
          if (q_last >= 0 && !mbar_wait(&sh->s_full[q_last & 1], (uint32_t)((q_last >> 1) & 1), limit_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            tmem_cp_128x256b(tmem + C::TM_Q + kk * 8, sw128_desc(q_addr + (kk / 4) * 16384 + (kk % 4) * 32, 16, 1024));
          SALAD_PROF(kPfQCopied);
        }
        if (n >= 1 && !issue_s()) { ok = false; break; }
        for (int j = 1; j < n && ok; ++j) {
          if (!issue_s() || !issue_pv(tt0 + j - 1, vj0 + j - 1, j == 1)) ok = false;
        }
        if (ok && n >= 1) ok = issue_pv(tt0 + n - 1, vj0 + n - 1, n == 1);
        if (!ok) break;
        tt += n;
        vj += n;
        if (im.lin && !issue_u(slot, seq)) { ok = false; break; }
        ++seq;
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
    // (running-max, rescale) decision; partial row sums are combined once per item.
    constexpr int HC = BLK / 2;                               // key columns per thread
    constexpr int HD = D / 2;                                 // feature columns per thread
    const int sw = warp - 2;
    const int hf = sw >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;                        // query row within the tile
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int half = BLK == 64 ? (r >> 6) : 0;               // query half (block 64), warp-uniform
    const uint64_t c2 = f32x2_pack(scale_log2, scale_log2);
    bool ok = true;
    int seq = 0, sj = 0, tt = 0, xc = 0;  // item, S slot, tile and exchange counters
    for (;;) {
      const int slot = seq & 1;
      if (!mbar_wait_warp(&sh->item_full[slot], (uint32_t)((seq >> 1) & 1), limit_ns)) { ok = false; break; }
      const Item im = sh->item[slot];
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->item_empty[slot]);
      if (im.w < 0) break;
      const uint32_t q_addr = sbase + C::OFF_Q0 + slot * C::Q_BYTES;
      float m_ref = -INFINITY;  // running reference max (raw score units), same in both halves
      float l = 0.f;            // this half's share of the row sum (of the bf16-rounded p)
      float le = 0.f;           // the same sum of the unrounded p, for the log-sum-exp output
      KeyIter it = item_iter(im, col_idx);  // read only when BLK == 64 (which rows use a tile)
      int j = 0;
      for (; j < im.n; ++j) {
        int bits = 1, vtile;
        if (BLK == 64) {
          int col;
          it.next(col, bits);
          vtile = min(BLK, N - col * BLK);
        } else {
          vtile = j == im.n - 1 ? im.vlast : BLK;  // only the last kept tile can be the partial block
        }
        const int s = sj & 1;
        const bool aborted = __shfl_sync(0xffffffffu, sh->abort_flag != 0, 0);
        SALAD_PROF(kPfSmWait);
        if (aborted || !mbar_wait_warp(&sh->s_full[s], (uint32_t)((sj >> 1) & 1), limit_ns)) { ok = false; break; }
        SALAD_PROF(kPfSmS);
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
        SALAD_PROF(kPfSmLoaded);

        const bool use = ((bits >> half) & 1) != 0;           // warp-uniform
        const int valid = vtile - hf * HC;  // real keys among this thread's columns (raster blocks)
        // (tile blocks: the tensor cores already put -inf on the slots past the grid)
        float mt;
        if (TILES || valid >= HC) {
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
        SALAD_PROF(kPfSmMax);
        // both halves of the row agree on the tile maximum (one barrier phase per
        // exchange; a bounded wait, so a time-out on either side cannot hang its partner)
        sh->xmax[xc & 1][hf][r] = mt;
        mbar_arrive(&sh->xbar[quarter]);
        if (!mbar_wait_warp(&sh->xbar[quarter], (uint32_t)(xc & 1), limit_ns)) { ok = false; break; }
        mt = fmaxf(mt, sh->xmax[xc & 1][hf ^ 1][r]);
        ++xc;
        SALAD_PROF(kPfSmXchg);
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
        // p = 2^(s * c - m_ref * c) in pairs; rows that do not use the tile write zeros.
        // The row sum adds the bf16-rounded p that the PV product consumes, so O / l
        // is a weighted mean with exactly the weights O was formed with: the rounding
        // of a dominant key's p (up to 2^8 under the lazy rescale) cancels in O / l.
        uint32_t pk[HC / 2];
        float rs, rse = 0.f;
        {
          const uint64_t nmb2 = f32x2_pack(-m_ref * scale_log2, -m_ref * scale_log2);
          uint64_t acc0 = 0, acc1 = 0, acc2 = 0, acc3 = 0;  // 0.0f pairs
          uint64_t acce = 0;
#pragma unroll
          for (int i = 0; i < HC / 2; ++i) {
            const uint64_t x =
                f32x2_fma(f32x2_pack(__uint_as_float(sr[2 * i]), __uint_as_float(sr[2 * i + 1])), c2, nmb2);
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
            pk[i] = pack_bf16x2(p0, p1);
            if (lse_out != nullptr) acce = f32x2_add(acce, f32x2_pack(p0, p1));
            const uint64_t pp = f32x2_pack(bf16_lo_to_f32(pk[i]), bf16_hi_to_f32(pk[i]));
            if ((i & 3) == 0) acc0 = f32x2_add(acc0, pp);
            if ((i & 3) == 1) acc1 = f32x2_add(acc1, pp);
            if ((i & 3) == 2) acc2 = f32x2_add(acc2, pp);
            if ((i & 3) == 3) acc3 = f32x2_add(acc3, pp);
          }
          const uint64_t a = f32x2_add(f32x2_add(acc0, acc1), f32x2_add(acc2, acc3));
          float a0, a1;
          f32x2_unpack(a, a0, a1);
          rs = a0 + a1;
          f32x2_unpack(acce, a0, a1);
          rse = a0 + a1;
        }
        if (!use) {
#pragma unroll
          for (int i = 0; i < HC / 2; ++i) pk[i] = 0u;
          rs = 0.f;
          rse = 0.f;
        }
        l = l * alpha + rs;
        le = le * alpha + rse;
        SALAD_PROF(kPfSmExp);
        // the P buffer and O were last read / written by the PV of global tile tt-1
        // (O is rescaled only within an item: an item's first tile has a reference
        // that starts at -inf)
        if (tt >= 1) {
          if (!mbar_wait_warp(&sh->pv_done[(tt - 1) & 1], (uint32_t)(((tt - 1) >> 1) & 1), limit_ns)) {
            ok = false;
            break;
          }
        }
        tc_fence_after();
        SALAD_PROF(kPfSmPv);
        if (j >= 1 && __any_sync(0xffffffffu, rescale)) {
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
        if constexpr (HC / 2 == 32) {
          tmem_st32(lane_addr + C::TM_P + hf * (HC / 2), *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        } else {
          tmem_st16(lane_addr + C::TM_P + hf * (HC / 2), *reinterpret_cast<uint32_t(*)[16]>(&pk[0]));
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sh->p_full[tt & 1]);
        SALAD_PROF(kPfSmP);
        ++sj;
        ++tt;
      }
      if (!ok) break;
      const int n = j;
      SALAD_PROF(kPfEpBegin);
      // relu(Q) over the Q columns of tensor memory for U, each thread its half of
      // its row, and this half's share of relu(q) . z on the way; the arrive
      // happens for every item, so the barrier keeps count of items
      float den_h = 0.f;
      // the Q buffer is overwritten by the output below: its load must be done
      // (an item with key tiles knows it through its first S, issued after it)
      if (n == 0 && !mbar_wait_warp(&sh->q_full[slot], (uint32_t)((seq >> 1) & 1), limit_ns)) {
        ok = false;
        break;
      }
      if (im.lin) {
        if (!mbar_wait_warp(&sh->z_full[slot], (uint32_t)((seq >> 1) & 1), limit_ns)) {
          ok = false;
          break;
        }
        // This half of the row of Q: from the Q columns of tensor memory, which hold
        // this item's Q (its S products are done: the last one completed before
        // this thread read its S); an item without key tiles never had its Q
        // copied there, so it reads the Q buffer in shared memory instead.
        constexpr int NP = C::DCH * 4;  // 16-byte pieces (8 features, 4 columns) in half a row
        uint32_t x[NP][4];
        const uint32_t q_cols = lane_addr + C::TM_Q + hf * 4 * NP;
        if (n >= 1) {
          if constexpr (NP == 8) {
            tmem_ld32(q_cols, *reinterpret_cast<uint32_t(*)[32]>(&x[0][0]));
          } else {
            tmem_ld16(q_cols, *reinterpret_cast<uint32_t(*)[16]>(&x[0][0]));
          }
          tmem_ld_wait();
        } else {
#pragma unroll
          for (int t = 0; t < NP; ++t) {
            const int piece = hf * NP + t;  // features 8 * piece ... 8 * piece + 7
            ld_shared_v4(q_addr + (piece / 8) * 16384 + sw128_offset((uint32_t)r, (uint32_t)(piece % 8)), x[t][0],
                         x[t][1], x[t][2], x[t][3]);
          }
        }
#pragma unroll
        for (int t = 0; t < NP; ++t)
#pragma unroll
          for (int i = 0; i < 4; ++i) x[t][i] = relu_bf16x2(x[t][i]);
        if constexpr (NP == 8) {
          tmem_st32(q_cols, *reinterpret_cast<uint32_t(*)[32]>(&x[0][0]));
        } else {
          tmem_st16(q_cols, *reinterpret_cast<uint32_t(*)[16]>(&x[0][0]));
        }
        const float4* zr = reinterpret_cast<const float4*>(sh->zs[slot]) + hf * NP * 2;
        float d0 = 0.f, d1 = 0.f;
#pragma unroll
        for (int t = 0; t < NP; ++t) {
          const float4 za = zr[2 * t], zb = zr[2 * t + 1];
          const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            d0 = fmaf(bf16_lo_to_f32(x[t][i]), zz[2 * i], d0);
            d1 = fmaf(bf16_hi_to_f32(x[t][i]), zz[2 * i + 1], d1);
          }
        }
        den_h = d0 + d1;
        tmem_st_wait();
        tc_fence_before();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sh->q_relu[slot]);
      SALAD_PROF(kPfEpRelu);
      if (n >= 1) {
        if (!mbar_wait_warp(&sh->pv_done[(tt - 1) & 1], (uint32_t)(((tt - 1) >> 1) & 1), limit_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
      }
      // the row sum and relu(q) . z of both halves
      sh->xsum[xc & 1][hf][r] = l;
      sh->xlse[xc & 1][hf][r] = le;
      sh->xden[xc & 1][hf][r] = den_h;
      mbar_arrive(&sh->xbar[quarter]);
      if (!mbar_wait_warp(&sh->xbar[quarter], (uint32_t)(xc & 1), limit_ns)) { ok = false; break; }
      l += sh->xsum[xc & 1][hf ^ 1][r];
      le += sh->xlse[xc & 1][hf ^ 1][r];
      const float gd = im.lin ? im.g / ((sh->xden[xc & 1][0][r] + sh->xden[xc & 1][1][r]) + eps) : 0.f;
      ++xc;
      SALAD_PROF(kPfEpSums);
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      if constexpr (!TILES) {
        // the row's log-sum-exp (natural log) of the sparse softmax, for training:
        // sum_j exp(scale s_j) = 2^(m_ref * scale * log2 e) * l
        if (lse_out != nullptr && hf == 0 && im.qtile * 128 + r < N)
          lse_out[(size_t)im.bh * N + im.qtile * 128 + r] =
              le > 0.f ? (m_ref * scale_log2 + log2f(le)) * 0.6931471805599453f : -INFINITY;
      }
      // U lands in the S slot after this item's tiles
      const int su = sj & 1;
      if (im.lin) {
        if (!mbar_wait_warp(&sh->s_full[su], (uint32_t)((sj >> 1) & 1), limit_ns)) { ok = false; break; }
        tc_fence_after();
      }
      SALAD_PROF(kPfEpU);
      // out = O / l + g U / den for this half's features -> bf16 staging in the Q buffer
      const uint32_t tm_u = su ? C::TM_S1 : C::TM_S0;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t ro[32], ru[32];
        if (n >= 1) {
          tmem_ld32(lane_addr + C::TM_O + hf * HD + c * 32, ro);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) ro[i] = 0u;
        }
        if (im.lin) {
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
      // O and U have been read: the next item's first PV and the S slot after U may proceed
      tc_fence_before();
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (im.lin) mbar_arrive(&sh->s_free[su]);
        mbar_arrive(&sh->staged[slot]);
      }
      SALAD_PROF(kPfEpEnd);
      if (im.lin) ++sj;
      ++seq;
    }
    if (!ok) record_timeout(sh, status);
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

template <int D, int BLK, bool TILES>
cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t s) {
  using C = AttnCfg<D, BLK>;
  const int smem = TILES ? C::SMEM_TILES : C::SMEM;
  cudaError_t e =
      cudaFuncSetAttribute(salad_attn_kernel<D, BLK, TILES>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  // a query tile is one raster tile of 128 rows, or one box
  const int qtiles = TILES ? (a.tiles.T / a.tiles.bt) * a.tiles.nh * a.tiles.nw : (a.N + 127) / 128;
  const long long items = (long long)qtiles * a.B * a.heads;
  int ctas = sm_count();
  if (a.max_ctas > 0 && a.max_ctas < ctas) ctas = a.max_ctas;
  const int grid = (int)(items < ctas ? items : ctas);
  salad_attn_kernel<D, BLK, TILES><<<grid, kThreads, smem, s>>>(
      *a.tm_q, *a.tm_k, *a.tm_v, *a.tm_out, *a.tm_t, a.row_ptr, a.col_idx, a.gate, a.z, a.heads, a.N, qtiles,
      (int)items, a.work_ctr, a.scale_log2, a.eps, a.status, a.wait_limit_ns, a.mask_per_bh, a.tiles, a.lse);
  return cudaGetLastError();
}

}  // namespace

// The profiling build's buffer: kProfRecorders x kProfEvents uint64 stamps per
// CTA, for the first bytes / (8 * kProfRecorders * kProfEvents) CTAs.
int set_profile_buffer(void* dev, size_t bytes) {
#ifdef SALAD_PROFILE
  const int ctas = (int)(bytes / (sizeof(uint64_t) * kProfRecorders * kProfEvents));
  uint64_t* p = static_cast<uint64_t*>(dev);
  if (cudaMemcpyToSymbol(g_prof_buf, &p, sizeof(p)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_prof_ctas, &ctas, sizeof(ctas)) != cudaSuccess)
    return SALAD_ERR_CUDA;
  return SALAD_OK;
#else
  (void)dev;
  (void)bytes;
  return SALAD_ERR_UNSUPPORTED;
#endif
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  if (a.tiles.bt > 0) return a.d == 64 ? launch_attn_t<64, 128, true>(a, s) : launch_attn_t<128, 128, true>(a, s);
  if (a.d == 64) return a.block == 64 ? launch_attn_t<64, 64, false>(a, s) : launch_attn_t<64, 128, false>(a, s);
  return a.block == 64 ? launch_attn_t<128, 64, false>(a, s) : launch_attn_t<128, 128, false>(a, s);
}

}  // namespace salad
