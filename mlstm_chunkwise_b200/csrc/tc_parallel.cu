// G3: intra-chunk TFLA kernel on tcgen05 (the parallel half of the chunkwise
// mLSTM forward pass), persistent.
//
// "Tiled Flash Linear Attention: More Efficient Linear RNN and xLSTM Kernels"
// (abstract): the intra-chunk part is tiled a second time, over query and
// key/value blocks, so the chunk size is not tied to the tile size.  A work
// item is 128 query rows (one L_Q tile) of one chunk and DVT value columns of
// one (b, h); it walks the L_KV = 128 key/value tiles of the chunk up to the
// diagonal.  For row r (token t) of chunk k with mu_r = max(m_k, amax_r):
//
//   O_r   = e^{m_k - mu_r} C_k^T q_r  +  sum_{s<=r} P_rs v_s
//   P_rs  = (s q_r.k_s) e^{acol_s - mu_r}                (0 above the diagonal)
//   den_r = e^{m_k - mu_r} n_k.q_r    +  sum_{s<=r} P_rs
//   h_r   = O_r / max(|den_r|, e^{-(bcum_r + mu_r)})
//
// The grid is at most one CTA per SM.  Items are numbered with the value tile
// fastest, then the query tile, then (b, h), and taken in rounds of gridDim.x
// consecutive items, so the CTAs running at the same time share chunks (K, V
// and the chunk state stay in L2).  Within a round the CTAs take the items in
// snake order (see item_at): an item's work grows with its query tile's
// position in the chunk, and the snake pairs heavy with light items.  The TMA
// producer runs ahead across item boundaries, so the next item's loads overlap
// the current item's P.V and epilogue.
//
// Roles (320 threads):
//   warp 0      TMA producer: Q tile per item, K / C / V slabs through a ring
//   warp 1      TMEM owner and single-thread MMA issuer
//   warps 2..9  two threads per query row (= TMEM lane), each owning half of
//               the columns: gating of S into P, rescaling of the inter-chunk
//               term, row sums, epilogue.
// TMEM (512 columns): the O accumulator at column 0 -- for DVT <= 128 a second
// one at column 128, used by alternate items so that one item's epilogue
// overlaps the next item's MMAs -- one S tile [128 x 128] at column 256 and two
// P buffers of 64 columns at 384 and 448.  The row threads load S_i, release
// the S buffer at once (so S_{i+1} is computed while they gate S_i), and write
// the gated tile as packed bf16 into P buffer i mod 2 (the half that owns keys
// [64h, 64h + 64) writes 32 packed columns at 32h), once the P.V MMA that read
// that buffer two tiles earlier has completed.  The P.V MMAs take their A
// operand from TMEM, so the gating of key tile i + 1 overlaps the P.V MMA of
// tile i and no MMA waits for another to complete.  With a single O buffer
// (value tiles of 256 columns) the epilogue stages each row's packed bf16
// output in the idle P buffers and releases O before its global stores, so the
// next item's inter-chunk MMAs overlap them.  Shared memory: the Q tile (DK/64
// swizzled slabs; two Q buffers at DK <= 128, so the next item's Q loads while
// this one runs), a ring of slabs as deep as the remaining space allows (at
// DK = 256: 9 stages of 16 KB for value tiles of up to 128 columns, 4 of 32 KB
// for 256, where two 16 KB K slabs share a stage), the per-item column weights
// and n_k.
// MMA order per item: S_0, Q.C, { S_i, P_{i-1}.V_{i-1} }, P_last.V_last.  When
// the tile works in one frame (see the row threads) P_0 is released as soon as
// it is written; otherwise the row threads gate S_0 while Q.C runs and rescale
// Q.C to the row frame before releasing P_0, so P_0.V_0 accumulates on the
// rescaled term.
#include <cuda.h>

#include "tc.h"
#include "tc_ptx.cuh"

namespace mlstm {
namespace {

using namespace tc;

constexpr int kThreads = 320;
constexpr int kQT = 128;  // query rows per item
constexpr int kKT = 128;  // key/value rows per intra tile
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 256;                 // O buffer(s) at columns 0 (and 128)
constexpr uint32_t kColP0 = 384, kColP1 = 448;  // two P buffers of 64 packed columns
constexpr uint32_t kColPHalf = 32;              // P columns of the upper key half
constexpr int kMaxL = 1024;  // largest chunk this kernel handles

template <int DK, int DVT>
struct Cfg {
  static_assert(DVT == 64 || DVT == 128 || DVT == 256, "value tile of 64, 128 or 256 columns");
  // Two O accumulators (alternating between items) fit next to the two S
  // buffers only for value tiles of at most 128 columns.
  static constexpr int kOBufs = DVT <= 128 ? 2 : 1;
  static constexpr int kSlabsK = DK / 64;
  static constexpr uint32_t kQBytes = kQT * DK * 2;
  // Two Q buffers where they cost at most two ring stages (d_qk <= 128): the
  // next item's Q and first slabs then load while this item still runs.
  static constexpr int kQBufs = DK <= 128 ? 2 : 1;
  static constexpr uint32_t kKSlabBytes = kKT * 128;           // 128 rows x 64 bf16
  static constexpr uint32_t kMNSlabBytes = (DVT / 64) * 8192;  // 64 rows x DVT bf16
  static constexpr uint32_t kStageBytes = kKSlabBytes > kMNSlabBytes ? kKSlabBytes : kMNSlabBytes;
  // K slabs per ring stage (two when a stage is sized for 256-column slabs)
  static constexpr int kKPer =
      (int)(kStageBytes / kKSlabBytes) < kSlabsK ? (int)(kStageBytes / kKSlabBytes) : kSlabsK;
  static_assert(kSlabsK % kKPer == 0, "K slabs fill whole stages");
  static constexpr uint32_t kMiscBytes = 2 * kMaxL * 4 + 2 * DK * 4 + 256 * 8 + 512;
  static constexpr uint32_t kBudget = 227 * 1024 - 1024;  // minus alignment slack
  static constexpr int kStagesFit =
      (int)((kBudget - kQBufs * kQBytes - kMiscBytes) / kStageBytes);
  static constexpr int kStages = kStagesFit > 12 ? 12 : kStagesFit;
  static_assert(kStages >= 3, "ring too shallow");
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffStage = kOffQ + kQBufs * kQBytes;
  static constexpr uint32_t kOffAcol = kOffStage + kStages * kStageBytes;  // float[2][kMaxL]
  static constexpr uint32_t kOffN = kOffAcol + 2 * kMaxL * 4;  // float[2][DK]
  static constexpr uint32_t kOffRed = kOffN + 2 * DK * 4;      // float2[256]
  static constexpr uint32_t kOffBar = kOffRed + 256 * 8;       // barriers
  static constexpr uint32_t kOffTmemSlot = kOffBar + 384;
  static constexpr uint32_t kBytes = kOffTmemSlot + 16;
  static constexpr uint32_t kSmem = kBytes + 1024;  // slack for 1024-byte alignment
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

// Barrier addresses, computed from one base (no arrays: a runtime-indexed
// array would live in local memory).
struct Bars {
  uint32_t a;
  __device__ __forceinline__ uint32_t full(int i) const { return a + 8 * i; }
  __device__ __forceinline__ uint32_t empty(int i) const { return a + 128 + 8 * i; }
  // per Q buffer: loaded; read by every MMA and row thread that needs it
  __device__ __forceinline__ uint32_t q_full(int b) const { return b ? a + 368 : a + 256; }
  __device__ __forceinline__ uint32_t q_empty(int b) const { return b ? a + 376 : a + 264; }
  // the S tile landed / was read; per P buffer: P written, P.V read it
  __device__ __forceinline__ uint32_t s_full() const { return a + 272; }
  __device__ __forceinline__ uint32_t s_empty() const { return a + 280; }
  __device__ __forceinline__ uint32_t p_full(int b) const { return a + 288 + 8 * b; }
  __device__ __forceinline__ uint32_t pv_done(int b) const { return a + 304 + 8 * b; }
  __device__ __forceinline__ uint32_t inter_done() const { return a + 320; }
  // per O buffer: accumulator complete, drained by the epilogue
  __device__ __forceinline__ uint32_t o_full(int b) const { return a + 328 + 8 * b; }
  __device__ __forceinline__ uint32_t o_empty(int b) const { return a + 344 + 8 * b; }
  __device__ __forceinline__ uint32_t mma_idle() const { return a + 360; }
};

// Work item -> (b*h, query tile, value tile).
struct Item {
  int bh, t0, dv0, k, c0, n_kv;
};

__device__ __forceinline__ Item decode_item(int it, const Problem& p, int n_dv, int n_q) {
  Item x;
  const int d = it % n_dv;
  const int rest = it / n_dv;
  const int qt = rest % n_q;
  x.bh = rest / n_q;
  x.t0 = qt * kQT;
  x.dv0 = d * (p.DV / n_dv);
  x.k = x.t0 / p.L;
  x.c0 = x.k * p.L;
  x.n_kv = (x.t0 - x.c0) / kKT + 1;
  return x;
}

// The k-th item of this CTA: round k, position c on even rounds and G - 1 - c
// on odd ones.  Item costs repeat with the period P = (query tiles per chunk)
// x (value tiles); when P divides 2G every CTA's pair of rounds sums to the
// same work (a plain stride gave each CTA the same position every round, and
// the kernel the time of the heaviest position).
__device__ __forceinline__ int item_at(int k) {
  const int G = (int)gridDim.x, c = (int)blockIdx.x;
  return k * G + ((k & 1) ? (G - 1 - c) : c);
}

template <int DK, int DVT>
__global__ void __launch_bounds__(kThreads, 1)
tc_parallel_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __nv_bfloat16* __restrict__ Cb,
                   Problem p, Gates g, const float* __restrict__ n_states,
                   __nv_bfloat16* __restrict__ H, float* __restrict__ n_out,
                   float* __restrict__ m_out, int n_items,
                   const __nv_bfloat16* __restrict__ Vraw) {
  using C = Cfg<DK, DVT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const Bars bar{sbase + C::kOffBar};
  float* acol_s = reinterpret_cast<float*>(smem + C::kOffAcol);
  float* n_s = reinterpret_cast<float*>(smem + C::kOffN);
  float2* red_s = reinterpret_cast<float2*>(smem + C::kOffRed);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + C::kOffTmemSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_dv = p.DV / DVT;
  const int n_q = (p.T + kQT - 1) / kQT;
  const long tpad = (long)p.NC * p.L;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::kStages; ++i) {
      mbar_init(bar.full(i), 1);
      mbar_init(bar.empty(i), 1);
    }
    for (int b = 0; b < C::kQBufs; ++b) {
      mbar_init(bar.q_full(b), 1);
      mbar_init(bar.q_empty(b), 1 + 256);  // MMA commit + the row threads' reads of Q
    }
    mbar_init(bar.s_full(), 1);
    mbar_init(bar.s_empty(), 256);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar.p_full(i), 256);
      mbar_init(bar.pv_done(i), 1);
      mbar_init(bar.o_full(i), 1);
      mbar_init(bar.o_empty(i), 256);
    }
    mbar_init(bar.inter_done(), 1);
    mbar_init(bar.mma_idle(), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32((const void*)tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------- TMA producer ----------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      int slab = 0;
      bool ok = true;
      auto next_stage = [&](uint32_t bytes) -> uint32_t {
        const int s = slab % C::kStages, u = slab / C::kStages;
        if (u > 0) ok = ok && mbar_wait(bar.empty(s), (u - 1) & 1, p, 1);
        mbar_expect_tx(bar.full(s), bytes);
        ++slab;
        return (uint32_t)s;
      };
      int n = 0;
      for (int it = item_at(0); it < n_items && ok; it = item_at(n + 1), ++n) {
        const Item x = decode_item(it, p, n_dv, n_q);
        auto load_k = [&](int i) {
          for (int c = 0; c < C::kSlabsK && ok; c += C::kKPer) {
            const uint32_t s = next_stage(C::kKPer * C::kKSlabBytes);
            for (int e = 0; e < C::kKPer; ++e)
              tma_load_3d(sbase + C::kOffStage + s * C::kStageBytes + e * C::kKSlabBytes, &tm_k,
                          (c + e) * 64, x.c0 + i * kKT, x.bh, bar.full(s));
          }
        };
        auto load_v = [&](int i) {
          for (int v = 0; v < 2 && ok; ++v) {
            const uint32_t s = next_stage(C::kMNSlabBytes);
            for (int b = 0; b < DVT / 64; ++b)
              tma_load_3d(sbase + C::kOffStage + s * C::kStageBytes + b * 8192, &tm_v,
                          x.dv0 + b * 64, x.c0 + i * kKT + v * 64, x.bh, bar.full(s));
          }
        };
        // Q before any ring slab of this item: the MMA consumes nothing of the
        // item until Q has landed, so a ring slab issued first could wait for
        // a stage that only frees after Q arrives.
        const int qb = n % C::kQBufs;
        if (n >= C::kQBufs) ok = mbar_wait(bar.q_empty(qb), ((n / C::kQBufs) - 1) & 1, p, 2);
        if (!ok) break;
        mbar_expect_tx(bar.q_full(qb), C::kQBytes);
        for (int c = 0; c < C::kSlabsK; ++c)
          tma_load_3d(sbase + C::kOffQ + qb * C::kQBytes + c * 16384, &tm_q, c * 64, x.t0, x.bh,
                      bar.q_full(qb));
        load_k(0);
        for (int c = 0; c < C::kSlabsK && ok; ++c) {
          const uint32_t s = next_stage(C::kMNSlabBytes);
          for (int b = 0; b < DVT / 64; ++b) {  // C_k rows [64c, 64c + 64) of block dv0 / 64 + b
            const size_t off =
                cb_block_row((long)x.bh * p.NC + x.k, x.dv0 / 64 + b, c * 64, DK, p.DV / 64);
            const bool in = MLSTM_IN_BOUNDS(p, off + 4096 <= (size_t)p.BH * p.NC * DK * p.DV);
            bulk_load(sbase + C::kOffStage + s * C::kStageBytes + b * 8192, Cb + (in ? off : 0),
                      8192, bar.full(s));
          }
        }
        for (int i = 1; i < x.n_kv && ok; ++i) {
          load_k(i);
          load_v(i - 1);
        }
        load_v(x.n_kv - 1);
      }
      // Drain: every issued load must have landed before the CTA may exit.
      for (int q = (slab > C::kStages ? slab - C::kStages : 0); q < slab; ++q)
        mbar_wait(bar.full(q % C::kStages), (q / C::kStages) & 1, p, 13);
      for (int m = (n > C::kQBufs ? n - C::kQBufs : 0); m < n; ++m)
        mbar_wait(bar.q_full(m % C::kQBufs), (m / C::kQBufs) & 1, p, 14);
    }
  } else if (warp == 1) {
    // ---------------------------- MMA issuer ------------------------------
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, kKT, 0, 0);
      constexpr uint32_t idO = idesc_bf16(128, DVT, 0, 1);
      bool ok = true;
      int slab = 0;   // ring position
      int tile = 0;   // S tiles issued so far (all items)
      uint32_t qoff = C::kOffQ;  // the current item's Q buffer
      auto take = [&]() -> uint32_t {
        const int s = slab % C::kStages, u = slab / C::kStages;
        ok = ok && mbar_wait(bar.full(s), u & 1, p, 5);
        tc_fence_after();
        ++slab;
        return (uint32_t)s;
      };
      // S tile j overwrites tile j - 1, which the row threads must have loaded.
      auto mma_s = [&]() {
        if (tile >= 1) ok = ok && mbar_wait(bar.s_empty(), (tile - 1) & 1, p, 4);
        tc_fence_after();
        const uint32_t d = tmem + kColS;
        for (int c = 0; c < C::kSlabsK; c += C::kKPer) {
          const uint32_t s = take();
          if (!ok) return;
          for (int e = 0; e < C::kKPer; ++e) {
            const uint32_t a0 = sbase + qoff + (c + e) * 16384;
            const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes + e * C::kKSlabBytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(d, sdesc_sw128(a0 + kk * 32, 16, 1024),
                          sdesc_sw128(b0 + kk * 32, 16, 1024), idS, (c | e | kk) != 0);
          }
          mma_commit(bar.empty(s));
        }
        mma_commit(bar.s_full());
        ++tile;
      };
      int ob = 0;  // output buffer of the current item
      // P_j . V_j with P_j (S tile j, gated) from P buffer j mod 2.
      auto mma_pv = [&](int j) {
        const int buf = j & 1;
        ok = ok && mbar_wait(bar.p_full(buf), (j >> 1) & 1, p, 7);
        tc_fence_after();
        const uint32_t aP = tmem + (buf ? kColP1 : kColP0);
        for (int v = 0; v < 2; ++v) {
          const uint32_t s = take();
          if (!ok) return;
          const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ts(tmem + ob * 128u, aP + (uint32_t)v * kColPHalf + (uint32_t)kk * 8u,
                        sdesc_sw128(b0 + kk * 2048, 8192, 1024), idO, 1);
          mma_commit(bar.empty(s));
        }
        mma_commit(bar.pv_done(buf));
      };
      int n = 0;
      for (int it = item_at(0); it < n_items && ok; it = item_at(n + 1), ++n) {
        const Item x = decode_item(it, p, n_dv, n_q);
        const int qb = n % C::kQBufs;
        qoff = C::kOffQ + qb * C::kQBytes;
        ok = mbar_wait(bar.q_full(qb), (n / C::kQBufs) & 1, p, 3);
        const int j0 = tile;  // this item's S_0
        if (ok) mma_s();
        // O buffers alternate between items (when there are two): the epilogue
        // of item n - kOBufs must have drained this one.
        ob = n % C::kOBufs;
        if (n >= C::kOBufs)
          ok = ok && mbar_wait(bar.o_empty(ob), ((n / C::kOBufs) - 1) & 1, p, 6);
        tc_fence_after();
        for (int c = 0; c < C::kSlabsK && ok; ++c) {  // inter-chunk term Q.C_k
          const uint32_t s = take();
          if (!ok) break;
          const uint32_t a0 = sbase + qoff + c * 16384;
          const uint32_t b0 = sbase + C::kOffStage + s * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + ob * 128u, sdesc_sw128(a0 + kk * 32, 16, 1024),
                        sdesc_sw128(b0 + kk * 2048, 8192, 1024), idO, (c | kk) != 0);
          mma_commit(bar.empty(s));
        }
        if (!ok) break;
        mma_commit(bar.inter_done());
        for (int i = 1; i < x.n_kv && ok; ++i) {
          mma_s();
          if (ok) mma_pv(j0 + i - 1);
        }
        if (!ok) break;
        mma_commit(bar.q_empty(qb));  // every MMA that reads Q has been issued
        mma_pv(j0 + x.n_kv - 1);
        if (!ok) break;
        mma_commit(bar.o_full(ob));
      }
      mma_commit(bar.mma_idle());  // completes once every MMA above has finished
      mbar_wait(bar.mma_idle(), 0, p, 15);
    }
  } else {
    // ------------------- gating / softmax / epilogue ----------------------
    // 256 row threads: half h = 0 (warps 2..5) owns S columns [0, 64), the
    // first DVT/2 output columns and the first half of the Q.n dot product;
    // half h = 1 (warps 6..9) owns the other halves.  Both halves of a row
    // combine their partial denominators once, in the epilogue.
    const int q = warp & 3;              // TMEM lane quadrant of this warp
    const int r = q * 32 + lane;         // query row in the tile = TMEM lane
    const int rt = threadIdx.x - 64;     // 0..255 among the row threads
    const int h = rt >> 7;               // column half
    const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
    const float ks = p.key_scale;
    // H rows go out in 32-byte stores where H allows it (row and tile starts
    // are then 32-byte aligned too: DV and every column offset are multiples
    // of 32 elements)
    const bool v8 = (reinterpret_cast<uintptr_t>(H) & 31) == 0;
    constexpr int kHalfO = DVT / 2;
    constexpr int kSlabsPerHalf = (C::kSlabsK + 1) / 2;
    bool ok = true;
    int tile = 0;
    int n = 0;

    // Per-item values, fetched one item ahead.  Every row's terms may be
    // scaled by a common factor, so when the exponents allow it (sep) the
    // whole tile works in one frame F instead of each row's mu_r:
    //   F = m_k, or the largest column weight c (amax of the tile's last row,
    //   amax being a running maximum) when no state enters the chunk (m_k =
    //   -inf), and
    //   P_rs = s (q_r.k_s) e^{acol_s - F},
    //   O_r  = e^{m_k - F} C_k^T q_r + sum_s P_rs v_s,   e^{m_k - F} = 1 or 0,
    //   h_r  = O_r / max(|den_r|, e^{-(bcum_r + F)}),
    // the row frame times e^{mu_r - F}.  Then P takes one column factor per
    // key (two lanes per packed multiply) and the inter-chunk term needs no
    // rescaling.  sep requires the column factors within e^60 of 1 (c - F, and
    // with F = c the first row's amax no lower than c - 60) and the floor's
    // exponent within +-80 over the tile's rows; otherwise every row keeps its
    // own frame, each element takes its own exponential (the column data holds
    // acol log2(e)) and the inter-chunk term is rescaled by e^{m_k - mu_r}.
    struct RowVals {
      float m_in, amax, bc, c, F;
      bool sep;
      int td;  // dominant token of the chunk's entering state, or -1
    };
    auto fetch_rows = [&](const Item& x) -> RowVals {
      RowVals v;
      const long base = (long)x.bh * tpad;
      v.m_in = g.mchk[(long)x.bh * (p.NC + 1) + x.k];
      v.amax = g.amax[base + x.t0 + r];
      v.bc = g.bcum[base + x.t0 + r];
      v.c = g.amax[base + x.t0 + kQT - 1];
      // uniform over the CTA: the same loads in every thread
      const bool fresh = v.m_in == -INFINITY;
      v.F = fresh ? v.c : v.m_in;
      const float spread = fresh ? v.c - g.amax[base + x.t0] : v.c - v.m_in;
      const float fl_hi = -g.bcum[base + x.t0 + kQT - 1] - v.F;  // bcum falls along the chunk
      const float fl_lo = -g.bcum[base + x.t0] - v.F;
      v.sep = spread <= 60.f && fl_hi <= 80.f && fl_lo >= -80.f;
      v.td = g.dom ? g.dom[(long)x.bh * p.NC + x.k] : -1;
      return v;
    };
    auto fetch_cols = [&](const Item& x, int buf, const RowVals& v) {
      float* ac = acol_s + buf * kMaxL;
      float* nn = n_s + buf * DK;
      for (int j = rt; j < x.n_kv * kKT; j += 256) {
        const float a = g.acol[(long)x.bh * tpad + x.c0 + j];
        ac[j] = v.sep ? ks * expf(a - v.F) : a * 1.4426950408889634f;  // -inf -> 0 / -inf
      }
      for (int j = rt; j < DK; j += 256) nn[j] = n_states[((long)x.bh * p.NC + x.k) * DK + j];
    };
    RowVals nx{0.f, 0.f, 0.f, 0.f, 0.f, false, -1};
    if (blockIdx.x < n_items) {
      const Item x0 = decode_item(blockIdx.x, p, n_dv, n_q);
      nx = fetch_rows(x0);
      fetch_cols(x0, 0, nx);
    }
    for (int it = item_at(0); it < n_items && ok; it = item_at(n + 1), ++n) {
      const Item x = decode_item(it, p, n_dv, n_q);
      const int t = x.t0 + r;
      const RowVals rv = nx;
      const float bc = rv.bc;
      const float* ac = acol_s + (n & 1) * kMaxL;
      const uint32_t colO = (uint32_t)(n % C::kOBufs) * 128u;
      const float* nn = n_s + (n & 1) * DK;
      const float mu = fmaxf(rv.m_in, rv.amax);  // the row's own frame
      const float fr = rv.sep ? rv.F : mu;        // the frame this tile works in
      const float mu2 = mu * 1.4426950408889634f;
      const float f_inter = expf(rv.m_in - fr);   // with sep: 1, or 0 with no entering state
      // The inter-chunk term is rescaled unless its factor is 1 (an m_k of
      // -inf still multiplies it by 0: a C0 given with m0 = -inf weighs nothing).
      const bool rescale = !rv.sep || rv.m_in == -INFINITY;
      named_bar_sync(1, 256);  // this item's column data is in shared memory

      // Partial den_inter = q_r . n_k over this half's slabs; then release Q.
      const int qb = n % C::kQBufs;
      ok = mbar_wait(bar.q_full(qb), (n / C::kQBufs) & 1, p, 8);
      float dn = 0.f;
      for (int c = h * kSlabsPerHalf; c < C::kSlabsK && c < (h + 1) * kSlabsPerHalf && ok; ++c) {
        const uint8_t* slab_ptr = smem + C::kOffQ + qb * C::kQBytes + c * 16384;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint4 v = *reinterpret_cast<const uint4*>(slab_ptr + sw128_offset(r, j));
          const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f2 = __bfloat1622float2(h2[e]);
            dn = fmaf(f2.x, nn[c * 64 + j * 8 + 2 * e], dn);
            dn = fmaf(f2.y, nn[c * 64 + j * 8 + 2 * e + 1], dn);
          }
        }
      }
      mbar_arrive(bar.q_empty(qb));
      float den = f_inter * dn;

      // Gated P tiles into the two TMEM P buffers (tile i into buffer i mod
      // 2).  P_0 is released only after this half of the inter-chunk term
      // (Q.C, issued after S_0) has been rescaled to the row frame mu_r, since
      // P_0.V_0 accumulates on top of it.
      for (int i = 0; i < x.n_kv; ++i, ++tile) {
        const int buf = tile & 1;
        ok = ok && mbar_wait(bar.s_full(), tile & 1, p, 10);
        tc_fence_after();
        const bool diag = (i == x.n_kv - 1);
        const uint32_t scol = kColS + h * 64;
        const uint32_t pcol = (buf ? kColP1 : kColP0) + h * kColPHalf;
        float rs = 0.f;
        {
          uint32_t v[64];
          tmem_ld32(trow + scol, *reinterpret_cast<uint32_t(*)[32]>(v));
          tmem_ld32(trow + scol + 32, *reinterpret_cast<uint32_t(*)[32]>(v + 32));
          tmem_wait_ld();
          tc_fence_before();
          mbar_arrive(bar.s_empty());  // S is in registers: the next S may land
          uint32_t pk[32];
          const float* acl = ac + i * kKT + h * 64;
          if (rv.sep && !diag) {
            uint64_t rs2 = 0;  // two fp32 partial sums, +0
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const float2 cf = *reinterpret_cast<const float2*>(acl + j);
              const uint64_t pp = mul_f32x2(
                  f32x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), f32x2(cf.x, cf.y));
              rs2 = add_f32x2(rs2, pp);
              const float2 pf = f32x2_split(pp);
              pk[j >> 1] = pack_bf16x2(pf.x, pf.y);
            }
            const float2 r2 = f32x2_split(rs2);
            rs = r2.x + r2.y;
          } else if (rv.sep) {
            uint64_t rs2 = 0;
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const int s0 = h * 64 + j;  // key/value index within the tile
              const float2 cf = *reinterpret_cast<const float2*>(acl + j);
              float2 pf = f32x2_split(mul_f32x2(
                  f32x2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])), f32x2(cf.x, cf.y)));
              if (s0 > r) pf.x = 0.f;
              if (s0 + 1 > r) pf.y = 0.f;
              rs2 = add_f32x2(rs2, f32x2(pf.x, pf.y));
              pk[j >> 1] = pack_bf16x2(pf.x, pf.y);
            }
            const float2 r2 = f32x2_split(rs2);
            rs = r2.x + r2.y;
          } else {
#pragma unroll
            for (int j = 0; j < 64; j += 2) {
              const int s0 = h * 64 + j;
              float pa = __uint_as_float(v[j]) * ks * ex2_approx(acl[j] - mu2);
              float pb = __uint_as_float(v[j + 1]) * ks * ex2_approx(acl[j + 1] - mu2);
              if (diag && s0 > r) pa = 0.f;
              if (diag && s0 + 1 > r) pb = 0.f;
              rs += pa + pb;
              pk[j >> 1] = pack_bf16x2(pa, pb);
            }
          }
          // P buffer buf was last read by the P.V MMAs of tile - 2
          if (tile >= 2) ok = ok && mbar_wait(bar.pv_done(buf), ((tile >> 1) - 1) & 1, p, 11);
          tc_fence_after();
          tmem_st32(trow + pcol, pk);
        }
        den += rs;
        if (!rescale && i == (x.n_kv > 1 ? 1 : 0)) {
          // Nothing to rescale, but the wait keeps this barrier's phases in
          // step: before P_1 (or the only P) is released, the MMA issuer
          // cannot have reached the next item's inter-chunk term.
          ok = ok && mbar_wait(bar.inter_done(), n & 1, p, 9);
          tc_fence_after();
        }
        if (rescale && i == 0) {
          ok = ok && mbar_wait(bar.inter_done(), n & 1, p, 9);
          tc_fence_after();
          if (ok) {
            for (int c = h * kHalfO; c < (h + 1) * kHalfO; c += 64) {
              uint32_t v0[32], v1[32];
              tmem_ld32(trow + colO + c, v0);
              if (kHalfO >= 64) tmem_ld32(trow + colO + c + 32, v1);
              tmem_wait_ld();
#pragma unroll
              for (int j = 0; j < 32; ++j)
                v0[j] = __float_as_uint(__uint_as_float(v0[j]) * f_inter);
              tmem_st32(trow + colO + c, v0);
              if (kHalfO >= 64) {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                  v1[j] = __float_as_uint(__uint_as_float(v1[j]) * f_inter);
                tmem_st32(trow + colO + c + 32, v1);
              }
            }
          }
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(bar.p_full(buf));
      }

      // Fetch the next item's row values and column data while P.V finishes.
      const int it_next = item_at(n + 1);
      if (it_next < n_items) {
        const Item xn = decode_item(it_next, p, n_dv, n_q);
        nx = fetch_rows(xn);
        fetch_cols(xn, (n + 1) & 1, nx);
      }

      // Epilogue: combine the two halves' denominators, h = O / max(|den|, e^{-m_r}),
      // with a dominated chunk's rank-one part (n_k^T q~_r) v_{t*} added in fp32.
      red_s[rt] = make_float2(den, dn);
      named_bar_sync(1, 256);
      const float2 other = red_s[rt ^ 128];
      den += other.x;
      const float c1 = f_inter * (dn + other.y);
      const __nv_bfloat16* vstar =
          rv.td >= 0 ? Vraw + ((long)x.bh * p.T + rv.td) * p.DV + x.dv0 : nullptr;
      ok = ok && mbar_wait(bar.o_full(n % C::kOBufs), (n / C::kOBufs) & 1, p, 12);
      tc_fence_after();
      const float mr = bc + fr;  // the floor's exponent in the tile's frame
      // the plain sigmoid variant has no normaliser: h = e^{m_r} O
      const float floor_f = expf(-mr);
      const float denom = p.no_norm ? floor_f : fmaxf(fabsf(den), floor_f);
      const float inv = p.no_norm ? expf(mr) : 1.f / denom;
      if constexpr (C::kOBufs == 1) {
        // One O buffer: this half's rows go as packed bf16 into its P buffer
        // (free: every P.V of the item has completed, and the next item's P is
        // written only after the row threads' barrier at its start), O is
        // released, and the global stores then read the staged rows, so the
        // next item's inter-chunk MMAs overlap them.
        const uint32_t stg = trow + (h ? kColP1 : kColP0);
        if (ok) {
#pragma unroll
          for (int c = 0; c < kHalfO; c += 32) {
            const int col = h * kHalfO + c;
            uint32_t v0[32], pk[16];
            tmem_ld32(trow + colO + col, v0);
            tmem_wait_ld();
            if (vstar) add_rank1_32(v0, c1, vstar + col);
#pragma unroll
            for (int j = 0; j < 32; j += 2)
              pk[j >> 1] =
                  pack_bf16x2(__uint_as_float(v0[j]) * inv, __uint_as_float(v0[j + 1]) * inv);
            tmem_st16(stg + c / 2, pk);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(bar.o_empty(0));
        if (ok) {
          // every lane reads (tcgen05.ld is warp-wide); rows past T store nothing
          const bool st = t < p.T &&
                          MLSTM_IN_BOUNDS(p, x.dv0 + (h + 1) * kHalfO <= p.DV && x.bh < p.BH);
          uint32_t* dst =
              reinterpret_cast<uint32_t*>(H + ((long)x.bh * p.T + t) * p.DV + x.dv0 + h * kHalfO);
#pragma unroll
          for (int c = 0; c < kHalfO / 2; c += 32) {
            uint32_t pk[32];
            tmem_ld32(stg + c, pk);
            tmem_wait_ld();
            if (st && v8) {  // whole 32-byte sectors
#pragma unroll
              for (int j = 0; j < 4; ++j) st_global_v8(dst + c + 8 * j, pk + 8 * j);
            } else if (st) {
#pragma unroll
              for (int j = 0; j < 8; ++j)
                reinterpret_cast<uint4*>(dst + c)[j] =
                    make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
          }
        }
      } else {
        if (ok) {
          for (int c = h * kHalfO; c < (h + 1) * kHalfO; c += 64) {
            uint32_t v0[32], v1[32];
            tmem_ld32(trow + colO + c, v0);
            if (kHalfO >= 64) tmem_ld32(trow + colO + c + 32, v1);
            tmem_wait_ld();
            if (vstar) {
              add_rank1_32(v0, c1, vstar + c);
              if (kHalfO >= 64) add_rank1_32(v1, c1, vstar + c + 32);
            }
            if (t < p.T && MLSTM_IN_BOUNDS(p, x.dv0 + c + (kHalfO >= 64 ? 64 : 32) <= p.DV &&
                                                  x.bh < p.BH)) {
              uint32_t pk[16];
#pragma unroll
              for (int j = 0; j < 32; j += 2)
                pk[j >> 1] =
                    pack_bf16x2(__uint_as_float(v0[j]) * inv, __uint_as_float(v0[j + 1]) * inv);
              uint4* dst =
                  reinterpret_cast<uint4*>(H + ((long)x.bh * p.T + t) * p.DV + x.dv0 + c);
              if (v8) {
                st_global_v8(dst, pk);
                st_global_v8(dst + 2, pk + 8);
              } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
              }
              if (kHalfO >= 64) {
#pragma unroll
                for (int j = 0; j < 32; j += 2)
                  pk[j >> 1] = pack_bf16x2(__uint_as_float(v1[j]) * inv,
                                           __uint_as_float(v1[j + 1]) * inv);
                if (v8) {
                  st_global_v8(dst + 4, pk);
                  st_global_v8(dst + 6, pk + 8);
                } else {
#pragma unroll
                  for (int j = 0; j < 4; ++j)
                    dst[4 + j] =
                        make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
                }
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(bar.o_empty(n % C::kOBufs));
      }
      if (t < p.T && x.dv0 == 0 && h == 0) {
        // per-token outputs in the row frame mu_r
        // (where the floor is picked, the row frame's floor itself, so that
        // a comparison with e^{-m_r} tells the two cases apart exactly)
        const float dr = !rv.sep ? denom
                         : (p.no_norm || !(fabsf(den) > floor_f)) ? expf(-(bc + mu))
                                                                  : fabsf(den) * expf(fr - mu);
        if (n_out) n_out[(long)x.bh * p.T + t] = p.signed_den ? copysignf(dr, den) : dr;
        if (m_out) m_out[(long)x.bh * p.T + t] = bc + mu;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

template <int DK, int DVT>
cudaError_t launch_parallel_t(const Problem& p, const void* Q, const void* K, const void* V,
                              Gates g, const __nv_bfloat16* Cb, const float* n_states, void* H,
                              float* n_out, float* m_out, cudaStream_t st) {
  using C = Cfg<DK, DVT>;
  CUtensorMap tq, tk, tv;
  if (!encode_tmap_bf16_3d(&tq, Q, p.DK, p.T, p.BH, 64, kQT) ||
      !encode_tmap_bf16_3d(&tk, K, p.DK, p.T, p.BH, 64, kKT) ||
      !encode_tmap_bf16_3d(&tv, V, p.DV, p.T, p.BH, 64, 64))
    return cudaErrorInvalidValue;
  auto kern = tc_parallel_kernel<DK, DVT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long items = (long)p.BH * ((p.T + kQT - 1) / kQT) * (p.DV / DVT);
  if (items > (1L << 30)) return cudaErrorInvalidValue;
  const int grid = (int)(items < sms ? items : sms);
  kern<<<grid, kThreads, C::kSmem, st>>>(tq, tk, tv, Cb, p, g, n_states,
                                         static_cast<__nv_bfloat16*>(H), n_out, m_out, (int)items,
                                         static_cast<const __nv_bfloat16*>(V));
  return cudaGetLastError();
}

}  // namespace

bool tc_parallel_supported(const Problem& p) {
  const bool dk_ok = p.DK == 64 || p.DK == 128 || p.DK == 256;
  const bool dv_ok = p.DV == 64 || p.DV == 128 || p.DV % 256 == 0;
  return dk_ok && dv_ok && p.DV <= 1024 && p.L % kKT == 0 && p.L <= kMaxL && p.T > 0;
}

cudaError_t launch_tc_parallel_bf16states(const Problem& p, const void* Q, const void* K,
                                          const void* V, Gates g, const __nv_bfloat16* Cb,
                                          const float* n_states, void* H, float* n_out,
                                          float* m_out, cudaStream_t st) {
  const int dvt = p.DV % 256 == 0 ? 256 : (p.DV >= 128 ? 128 : p.DV);
#define MLSTM_PAR_CASE(dk, dvt_)                                                                \
  if (p.DK == dk && dvt == dvt_)                                                                \
    return launch_parallel_t<dk, dvt_>(p, Q, K, V, g, Cb, n_states, H, n_out, m_out, st);
  MLSTM_PAR_CASE(64, 64)
  MLSTM_PAR_CASE(64, 128)
  MLSTM_PAR_CASE(64, 256)
  MLSTM_PAR_CASE(128, 64)
  MLSTM_PAR_CASE(128, 128)
  MLSTM_PAR_CASE(128, 256)
  MLSTM_PAR_CASE(256, 64)
  MLSTM_PAR_CASE(256, 128)
  MLSTM_PAR_CASE(256, 256)
#undef MLSTM_PAR_CASE
  return cudaErrorNotSupported;
}

}  // namespace mlstm
